// Forward pass on the tensor cores (sm_100a): tcgen05.mma with TMEM
// accumulators, TMA-staged tiles, online softmax.
//
// Computes O_i = softmax(scale q_i K_{S_i}^T) V_{S_i} and LSE_i over the live
// tiles of each query tile ("Sparse Transformer", llm-arch-kb, section 2,
// "Per-layer cost": a block-sparse matmul over the pattern's blocks; the
// milestone page, "The notation", for the attention itself).
//
// Persistent CTAs, two per SM (96 KB shared memory and 256 TMEM columns
// each, so the two CTAs of an SM interleave their MMA and softmax phases).
// Work units (query tile x head, longest first) are claimed from a counter
// by warp 4, decoded once (item and head) and published to the other roles
// through a shared-memory ring, so a CTA takes the next unit when it is
// ready for one. The counter is one of the layout's slots; the last CTA to
// finish resets it. The second pass of a two-pass layout is a separate
// instantiation (MERGE) that merges into the first pass's O and LSE; one-pass
// launches carry no merge code. Warp roles:
//   warp 4       TMA producer: claims the units; each unit's Q tile into one
//                of two Q buffers (the next unit's Q loads while the current
//                one computes) and K tiles into a 2-stage ring released by the
//                S MMA;
//   warp 6       TMA producer: V tiles into a 2-stage ring released by PV
//                (natural, summary or residue-class view for both);
//   warp 5       TMEM owner and MMA issuer: S = Q K^T (M=128, N=128, K=64)
//                into TMEM, then O += P V with P read from TMEM (A operand)
//                and V from shared memory (MN-major);
//   warps 0..3   softmax: thread = query row = TMEM lane. Loads S, applies the
//                row's live-key interval on PARTIAL tiles, keeps the running
//                max (rescaling O in TMEM only when the max grows by more than
//                2^8) and sum, writes P as bf16 pairs into TMEM; at the end of
//                a unit normalises O, merges with the first pass (MERGE), and
//                stores O (32-byte stores when the output allows) and LSE
//                from registers.
// Every wait is bounded; a wait that runs out sets the status word, raises
// the CTA's abort flag, and all roles drain their in-flight work and return.
#include <math.h>

#include <algorithm>

#include "launch.h"
#include "tc_common.cuh"

namespace st {
namespace {

using namespace tc;

constexpr int NS = 2;                       // K/V stages
constexpr int kSched = 4;                   // published work units in flight
constexpr int kTileBytes = kTile * 64 * 2;  // one 128 x 64 bf16 tile
constexpr int kThreads = 256;  // warpgroup 0: softmax; warpgroup 1: TMA, MMA
constexpr uint32_t kRegsSoftmax = 208, kRegsIssue = 48;
static_assert(128 * kRegsSoftmax + 128 * kRegsIssue == kThreads * 128, "register split");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct FwdMaps {
  CUtensorMap q[3], k[3], v[3];  // indexed by View
};

struct SmemFwd {
  uint8_t q[2][kTileBytes];
  uint8_t k[NS][kTileBytes];
  uint8_t v[NS][kTileBytes];
  uint64_t q_full[2], q_empty[2], k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full, s_free, p_full, pv_done, o_free, fin;
  uint64_t sched_full[kSched], sched_empty[kSched];
  // published work units: index (n_units: no more work), head, item; the
  // producer decodes each unit once and the other roles read it from here
  int sched_u[kSched], sched_bh[kSched];
  FwdItem sched_it[kSched];
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

// Live key columns [lo, hi) of key tile `ke` for the query at natural
// position i, with blk = i / l (its block, or in the residue view its class
// row). The bounds restate the segment rules as intervals.
__device__ __forceinline__ void live_cols(const Geom& g, const KeyEnt& ke, int i, int blk,
                                          int& lo, int& hi) {
  if (i < 0) {
    lo = hi = 0;
    return;
  }
  const int l = g.l, c = g.c;
  int a = 0, b = 0, base = 0, lim = 0;
  if (ke.kview == VIEW_NAT) {
    base = ke.ktile * kTile;
    lim = g.T;
    switch (ke.rule) {
      case RULE_CAUSAL: a = 0; b = i + 1; break;
      case RULE_BAND: a = max(0, i - l); b = i + 1; break;
      case RULE_BLOCK: a = blk * l; b = i + 1; break;
      case RULE_STRIDE: a = i; b = i + 1; break;          // natural keys only when l >= T
      case RULE_SUMMARY: a = l - c; b = i + 1; break;     // natural keys only when l >= T
      default: a = 0; b = 0; break;                        // stride_far / summary_earlier: empty
    }
  } else if (ke.kview == VIEW_SUM) {
    base = ke.ktile * kTile;
    lim = g.nsum;
    const int off = i - blk * l;
    a = 0;
    b = blk * c + ((ke.rule == RULE_SUMMARY) ? max(0, off - (l - c) + 1) : 0);
  } else {
    // key tile column x holds view row ktile * 128 + x; the query's class r
    // starts at view row r * cw
    base = ke.ktile * kTile - (i - blk * l) * g.cw;
    lim = g.P;
    a = 0;
    b = (ke.rule == RULE_STRIDE) ? blk + 1 : blk - 1;
  }
  b = min(b, lim);
  lo = max(a - base, 0);
  hi = min(b - base, kTile);
  if (hi < lo) hi = lo;
}

struct Unit {
  FwdItem it;
  int bh;
};

__device__ __forceinline__ Unit unit_of(const FwdItem* items, int u, int NH, const Heads& hs) {
  Unit x;
  const int q = fdiv(u, hs.fnh);  // NH = the divisor of hs.fnh
  x.it = items[q];
  x.bh = head_of(u - q * NH, x.it.hclass, hs);
  return x;
}

// F16: 16-bit element type (fp16 if true, else bf16). MERGE: the launch is
// the second pass of a two-pass layout and merges its result into the O and
// LSE already in the outputs (a separate instantiation, so that one-pass
// launches carry no merge code).
template <bool F16, bool MERGE, bool PACKED>
__global__ void __launch_bounds__(kThreads, 2)
fwd_tc_kernel(const __grid_constant__ FwdMaps maps, Geom g, const FwdItem* __restrict__ items,
              int n_units, int NH, const KeyEnt* __restrict__ keys, Heads hs,
              float scale_log2, uint16_t* __restrict__ out, float* __restrict__ lse,
              int* sched_slot, int* status, uint64_t wait_ns, int force_timeout) {
  extern __shared__ uint8_t smem_raw[];
  SmemFwd& S = *reinterpret_cast<SmemFwd*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.q_full[b], 1);
      mbar_init(&S.q_empty[b], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.k_full[s], 1);
      mbar_init(&S.k_empty[s], 1);
      mbar_init(&S.v_full[s], 1);
      mbar_init(&S.v_empty[s], 1);
    }
    mbar_init(&S.s_full, 1);
    mbar_init(&S.s_free, 128);
    mbar_init(&S.p_full, 128);
    mbar_init(&S.pv_done, 1);
    mbar_init(&S.o_free, 128);
    mbar_init(&S.fin, 1);
    for (int k = 0; k < kSched; ++k) {
      mbar_init(&S.sched_full[k], 1);
      mbar_init(&S.sched_empty[k], 6);  // V producer, MMA lane, 4 softmax warps
    }
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 7) {  // the tensor maps into the descriptor cache, one per lane
    const CUtensorMap* m = &maps.q[0];
    if (lane < (int)(sizeof(FwdMaps) / sizeof(CUtensorMap))) tma_prefetch_desc(m + lane);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  auto fail = [&]() {
    *abort = 1;
    set_status(status, ST_ERR_DEVICE_TIMEOUT);
  };
  // Next published unit for a consuming role (one arrival per consuming warp).
  int sk = 0;
  auto next_unit = [&](int& u, Unit& x, bool arrive) -> bool {
    const int k = sk % kSched;
    if (!mbar_wait(&S.sched_full[k], (sk / kSched) & 1, wait_ns, abort)) return false;
    u = *reinterpret_cast<volatile int*>(&S.sched_u[k]);
    x.it = S.sched_it[k];
    x.bh = S.sched_bh[k];
    if (arrive) mbar_arrive(&S.sched_empty[k]);
    ++sk;
    return true;
  };

  // Registers: the launch gives 128 per thread; the softmax warpgroup raises
  // its budget to kRegsSoftmax and the TMA / MMA warpgroup lowers its own to
  // kRegsIssue (128 * kRegsSoftmax + 128 * kRegsIssue = 256 * 128). Each
  // role's whole body sits inside the branch that set its budget.
  if (warp >= 4) {
    regs_decrease<kRegsIssue>();
  if (warp == 4) {
    // ---------------- TMA producer: Q and K ----------------
    if (lane == 0) {
      int kv_last[NS] = {-1, -1};
      int q_last[2] = {-1, -1};
      int gt = 0;  // global tile counter of this CTA
      bool ok = true;
      int n = 0, pub = 0;
      // Unit u of the CTA's first is blockIdx.x (the longest units spread one
      // per CTA); later ones come from the counter, offset by the grid.
      // The first valid unit at or after u (n_units if none), decoded into y.
      auto valid = [&](int u, Unit& y) -> int {
        for (;;) {
          if (u >= n_units) return n_units;
          y = unit_of(items, u, NH, hs);
          if (y.bh >= 0) return u;
          u = (int)gridDim.x + atomicAdd(sched_slot, 1);
        }
      };
      auto publish = [&](int u, const Unit& y) -> bool {
        const int k = pub % kSched;
        if (!mbar_wait(&S.sched_empty[k], ((pub / kSched) & 1) ^ 1, wait_ns, abort)) return false;
        S.sched_u[k] = u;
        if (u < n_units) {
          S.sched_it[k] = y.it;
          S.sched_bh[k] = y.bh;
        }
        mbar_arrive(&S.sched_full[k]);
        ++pub;
        return true;
      };
      Unit x;
      int cur = valid(blockIdx.x, x);
      while (ok && cur < n_units) {
        if (!publish(cur, x)) {
          ok = false;
          break;
        }
        // the claim of the following unit goes out now, answered by the end
        const int ticket = (int)gridDim.x + atomicAdd(sched_slot, 1);
        const int qb = n & 1;
        if (!mbar_wait(&S.q_empty[qb], ((n >> 1) & 1) ^ 1, wait_ns, abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&S.q_full[qb], kTileBytes);
        load_tile<PACKED>(S.q[qb], maps.q, x.it.qview, g, x.it.qtile, x.bh, &S.q_full[qb]);
        q_last[qb] = n;
        for (int e = x.it.kbeg; e < x.it.kend; ++e, ++gt) {
          const int s = gt % NS;
          if (!mbar_wait(&S.k_empty[s], ((gt / NS) & 1) ^ 1, wait_ns, abort)) {
            ok = false;
            break;
          }
          if (force_timeout && gt == 0) continue;  // test hook: this stage never fills
          const KeyEnt ke = keys[e];
          mbar_arrive_expect_tx(&S.k_full[s], kTileBytes);
          load_tile<PACKED>(S.k[s], maps.k, ke.kview, g, ke.ktile, x.bh, &S.k_full[s]);
          if (e + 2 < x.it.kend) {
            const KeyEnt kn = keys[e + 2];
            prefetch_tile<PACKED>(maps.k, kn.kview, g, kn.ktile, x.bh);
          }
          kv_last[s] = gt;
        }
        ++n;
        cur = valid(ticket, x);
      }
      if (ok && !publish(n_units, x)) ok = false;  // no more work
      if (!ok) fail();
      // no copy may be in flight when the CTA exits (these waits ignore the
      // abort flag: the copies were issued and will land)
      for (int b = 0; b < 2; ++b)
        if (q_last[b] >= 0 && !mbar_wait_drain(&S.q_full[b], (q_last[b] >> 1) & 1, wait_ns))
          fail();
      for (int s = 0; s < NS; ++s)
        if (kv_last[s] >= 0 && !mbar_wait_drain(&S.k_full[s], (kv_last[s] / NS) & 1, wait_ns))
          fail();
    }
  } else if (warp == 6) {
    // ---------------- TMA producer: V (its own ring, freed by PV) ----------------
    if (lane == 0) {
      int v_last[NS] = {-1, -1};
      int gt = 0;
      bool ok = true;
      for (;;) {
        int u = 0;
        Unit x;
        if (!next_unit(u, x, true)) {
          ok = false;
          break;
        }
        if (u >= n_units) break;
        for (int e = x.it.kbeg; e < x.it.kend; ++e, ++gt) {
          const int s = gt % NS;
          if (!mbar_wait(&S.v_empty[s], ((gt / NS) & 1) ^ 1, wait_ns, abort)) {
            ok = false;
            break;
          }
          const KeyEnt ke = keys[e];
          mbar_arrive_expect_tx(&S.v_full[s], kTileBytes);
          load_tile<PACKED>(S.v[s], maps.v, ke.kview, g, ke.ktile, x.bh, &S.v_full[s]);
          if (e + 2 < x.it.kend) {  // two tiles ahead of the ring: into L2 now
            const KeyEnt kn = keys[e + 2];
            prefetch_tile<PACKED>(maps.v, kn.kview, g, kn.ktile, x.bh);
          }
          v_last[s] = gt;
        }
      }
      if (!ok) fail();
      for (int s = 0; s < NS; ++s)
        if (v_last[s] >= 0 && !mbar_wait_drain(&S.v_full[s], (v_last[s] / NS) & 1, wait_ns))
          fail();
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idS = idesc_16(128, 128, false, false, F16);
      const uint32_t idPV = idesc_16(128, 64, false, true, F16);
      bool ok = true;
      int gt = 0, n = 0;  // tiles and units of this CTA issued so far
      // S of global tile g from Q buffer qb and K ring stage g % NS.
      auto issue_s = [&](int g, int qb) -> bool {
        const int s = g % NS;
        if (!mbar_wait(&S.k_full[s], (g / NS) & 1, wait_ns, abort)) return false;
        tc_fence_after();
        const uint64_t qd = sdesc(smem_u32(S.q[qb]), 16, 1024);
        const uint64_t kd = sdesc(smem_u32(S.k[s]), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + kColS, sdesc_at(qd, kk * 32), sdesc_at(kd, kk * 32), idS, kk > 0);
        mma_commit(&S.s_full);
        mma_commit(&S.k_empty[s]);
        return true;
      };
      Unit cur, nx;
      int u = n_units, un = n_units;
      ok = next_unit(u, cur, true);
      bool first_done = false;  // S of this unit's first tile already issued ahead
      while (ok && u < n_units) {
        const int qb = n & 1;
        const int cnt = cur.it.kend - cur.it.kbeg;
        if (!mbar_wait(&S.q_full[qb], (n >> 1) & 1, wait_ns, abort)) {
          ok = false;
          break;
        }
        if (cnt > 0 && !first_done) {
          if (gt > 0 && !mbar_wait(&S.s_free, (gt - 1) & 1, wait_ns, abort)) {
            ok = false;
            break;
          }
          if (!issue_s(gt, qb)) {
            ok = false;
            break;
          }
        }
        first_done = false;
        bool have_next = false;  // the following unit has been read from the ring
        for (int e = 0; e < cnt; ++e, ++gt) {
          const int s = gt % NS;
          // The following unit is read from the ring at this unit's last tile:
          // by then all of this unit's K tiles have been issued, so the
          // producer has published it.
          if (e + 1 == cnt) {
            if (!next_unit(un, nx, true)) {
              ok = false;
              break;
            }
            have_next = true;
          }
          // S of the next tile (this unit's, or the first of the next unit) goes
          // out as soon as the softmax has read S of this one, ahead of PV.
          const bool next_here = (e + 1 < cnt);
          const bool next_unit = !next_here && un < n_units && nx.it.kend > nx.it.kbeg;
          if (next_here || next_unit) {
            if (!mbar_wait(&S.s_free, gt & 1, wait_ns, abort)) {
              ok = false;
              break;
            }
            int nqb = qb;
            if (next_unit) {
              nqb = (n + 1) & 1;
              if (!mbar_wait(&S.q_full[nqb], ((n + 1) >> 1) & 1, wait_ns, abort)) {
                ok = false;
                break;
              }
            }
            if (!issue_s(gt + 1, nqb)) {
              ok = false;
              break;
            }
            if (next_unit) first_done = true;
          }
          if (!mbar_wait(&S.p_full, gt & 1, wait_ns, abort)) {
            ok = false;
            break;
          }
          if (e == 0 && !mbar_wait(&S.o_free, (n & 1) ^ 1, wait_ns, abort)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&S.v_full[s], (gt / NS) & 1, wait_ns, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vd = sdesc(smem_u32(S.v[s]), 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kColO, tmem + kColP + kk * 8, sdesc_at(vd, kk * 2048),
                   idPV, (e > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&S.pv_done);
          mma_commit(&S.v_empty[s]);
        }
        if (!ok) break;
        if (!have_next) {  // a unit without tiles
          if (!next_unit(un, nx, true)) {
            ok = false;
            break;
          }
        }
        mma_commit(&S.q_empty[qb]);
        ++n;
        u = un;
        cur = nx;
      }
      if (!ok) fail();
      // every MMA issued has completed before TMEM is freed
      mma_commit(&S.fin);
      if (!mbar_wait_drain(&S.fin, 0, wait_ns)) fail();
    }
  }
  } else {
    regs_increase<kRegsSoftmax>();
    // ---------------- softmax warps ----------------
    const int lg = warp;              // TMEM lane group of this warp
    const int row = lg * 32 + lane;   // query row in the tile = TMEM lane
    const uint32_t tl = (uint32_t)(lg * 32) << 16;
    bool ok = true;
    int gt = 0, n = 0;
    // A unit's epilogue (O / l, merge, stores) runs inside the next unit's
    // first tile: after that tile's exponentials, at the point where the last
    // PV of the unit has to be complete anyway before P is overwritten.
    struct Pending {
      int i, bh, cnt, merge;
      float m, l;
    };
    Pending pend = {-1, 0, 0, 0, 0.f, 0.f};
    bool pending = false;
    // part 1: O out of TMEM (then the accumulator is free for the next unit)
    auto load_o = [&](const Pending& pe, float* o) {
#pragma unroll
      for (int xk = 0; xk < 64; ++xk) o[xk] = 0.f;
      if (pe.cnt > 0) {
        tmem_ld32(tmem + tl + kColO, reinterpret_cast<uint32_t*>(o));
        tmem_ld32(tmem + tl + kColO + 32, reinterpret_cast<uint32_t*>(o) + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&S.o_free);
    };
    // part 2: normalise, merge with a previous pass, store O and LSE
    auto finish_o = [&](const Pending& pe, float* o) {
      if (pe.i < 0) return;
      const float inv = (pe.l > 0.f) ? 1.f / pe.l : 0.f;
      float L = (pe.l > 0.f) ? (pe.m + __log2f(pe.l)) * 0.69314718055994531f : -INFINITY;
#pragma unroll
      for (int xk = 0; xk < 64; ++xk) o[xk] *= inv;
      const size_t rowoff = ((size_t)pe.bh * g.T + pe.i) * 64;
      uint4* dst = reinterpret_cast<uint4*>(out + rowoff);
      if constexpr (MERGE) {
        const float Lp = lse[(size_t)pe.bh * g.T + pe.i];
        const float mx2 = fmaxf(Lp, L);
        float wp = 0.f, wc = 0.f;
        if (mx2 != -INFINITY) {
          const float Ln = mx2 + __logf(__expf(Lp - mx2) + __expf(L - mx2));
          wp = __expf(Lp - Ln);
          wc = __expf(L - Ln);
          L = Ln;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint4 w = dst[ch];
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const float2 f = unpack2<F16>(ws[q2]);
            o[ch * 8 + 2 * q2] = fmaf(wp, f.x, wc * o[ch * 8 + 2 * q2]);
            o[ch * 8 + 2 * q2 + 1] = fmaf(wp, f.y, wc * o[ch * 8 + 2 * q2 + 1]);
          }
        }
      }
      uint32_t w[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) w[x] = pack2<F16>(o[2 * x], o[2 * x + 1]);
      // the row leaves in whole 32-byte sectors when the output allows it
      // (rows are 128 bytes, so all rows share the base's alignment)
      if ((reinterpret_cast<uintptr_t>(out) & 31) == 0) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) st_global_v8(dst + 2 * ch, w + 8 * ch);
      } else {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          dst[ch] = make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
      }
      lse[(size_t)pe.bh * g.T + pe.i] = L;
    };
    auto epilogue = [&](const Pending& pe) {
      float o[64];
      load_o(pe, o);
      finish_o(pe, o);
    };
    for (;;) {
      int u = 0;
      Unit x;
      const bool got = next_unit(u, x, false);
      __syncwarp();
      if (lane == 0 && got) mbar_arrive(&S.sched_empty[(sk - 1) % kSched]);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const bool end = u >= n_units;
      if (end) {
        x.it = FwdItem{0, 0, 0, 0, 0, 0, 0};
        x.bh = 0;
      }
      const FwdItem& it = x.it;
      const int i = end ? -1 : view_pos(g, it.qview, it.qtile, row);
      const int iblk = i >= 0 ? fdiv(i, g.fl) : 0;
      const int cnt = it.kend - it.kbeg;
      if (end || cnt == 0) {
        // the pending unit's output goes out here (one copy of the epilogue
        // for empty units and for the end of the work); an empty unit then
        // becomes the pending one, written by the next flush
        if (pending) {
          if (gt > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&S.pv_done, (gt - 1) & 1, wait_ns, abort));
            if (!ok) break;
            tc_fence_after();
          }
          epilogue(pend);
          pending = false;
        }
        if (end) break;
        pend = {i, x.bh, 0, (int)it.merge, -INFINITY, 0.f};
        pending = true;
        ++n;
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int e = 0; e < cnt; ++e, ++gt) {
        const KeyEnt ke = keys[it.kbeg + e];
        ok = __all_sync(0xffffffffu, mbar_wait(&S.s_full, gt & 1, wait_ns, abort));
        if (!ok) break;
        tc_fence_after();
        // S is read from TMEM once; the buffer is released at once so the MMA
        // warp can compute the next tile's S while this one is exponentiated.
        // FULL tiles skip the per-element mask.
        float s[128];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          tmem_ld32(tmem + tl + kColS + c4 * 32, reinterpret_cast<uint32_t*>(s) + c4 * 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&S.s_free);
        const bool full = (ke.flag == TILE_FULL);
        if (!full) {
          int lo, hi;
          live_cols(g, ke, i, iblk, lo, hi);
          mask_cols<4>(s, 0, lo, hi);
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int xk = 0; xk < 128; xk += 8) {
          m4[0] = fmax3(m4[0], s[xk + 0], s[xk + 1]);
          m4[1] = fmax3(m4[1], s[xk + 2], s[xk + 3]);
          m4[2] = fmax3(m4[2], s[xk + 4], s[xk + 5]);
          m4[3] = fmax3(m4[3], s[xk + 6], s[xk + 7]);
        }
        const float mt = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * scale_log2;
        const float m_new = fmaxf(m_run, mt);
        float alpha = 1.f;
        bool rescale_o = false;
        if (m_new > m_run + kRescaleThreshold) {
          rescale_o = (m_run != -INFINITY);
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        const float mu = (m_run == -INFINITY) ? 0.f : m_run;
        // exponentials: one packed FMA forms two exponents, masked entries are
        // -inf and give exactly 0; four pairs of partial sums break the add chain
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        const float nmu = -mu;
        uint32_t pk[64];
#pragma unroll
        for (int xk = 0; xk < 128; xk += 2) {
          float a0, a1;
          ffma2(a0, a1, s[xk], s[xk + 1], scale_log2, scale_log2, nmu, nmu);
          const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
          const int j = (xk >> 1) & 3;
          fadd2(sa[j], sb[j], sa[j], sb[j], p0, p1);
          pk[xk >> 1] = pack2<F16>(p0, p1);
        }
        l_run = l_run * alpha + (((sa[0] + sb[0]) + (sa[1] + sb[1])) +
                                 ((sa[2] + sb[2]) + (sa[3] + sb[3])));
        if (gt > 0) {
          // PV of the previous tile is done: P may be overwritten, O is stable
          ok = __all_sync(0xffffffffu, mbar_wait(&S.pv_done, (gt - 1) & 1, wait_ns, abort));
          if (!ok) break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, rescale_o)) {
          const float a = rescale_o ? alpha : 1.f;
#pragma unroll 1
          for (int c8 = 0; c8 < 8; ++c8) {
            uint32_t o[8];
            tmem_ld8(tmem + tl + kColO + c8 * 8, o);
            tmem_wait_ld();
#pragma unroll
            for (int xk = 0; xk < 8; ++xk) o[xk] = __float_as_uint(__uint_as_float(o[xk]) * a);
            tmem_st8(tmem + tl + kColO + c8 * 8, o);
          }
        }
        tmem_st32(tmem + tl + kColP, pk);
        tmem_st32(tmem + tl + kColP + 32, pk + 32);
        tmem_wait_st();
        // the previous unit's O leaves TMEM before this unit's first PV may
        // start; its normalisation and stores overlap that PV
        if (e == 0 && pending) {
          float o[64];
          load_o(pend, o);
          tc_fence_before();
          mbar_arrive(&S.p_full);
          finish_o(pend, o);
          pending = false;
        } else {
          tc_fence_before();
          mbar_arrive(&S.p_full);
        }
      }
      if (!ok) break;
      pend = {i, x.bh, cnt, (int)it.merge, m_run, l_run};
      pending = true;
      ++n;
    }
    if (!ok) fail();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
  // the last CTA out resets the work counter for the slot's next launch
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(sched_slot + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(sched_slot, 0);
      atomicExch(sched_slot + 1, 0);
    }
  }
}

}  // namespace

namespace {

template <bool F16>
cudaError_t tc_fwd_t(const Call& c, const void* q, const void* k, const void* v, void* o,
                     float* lse, int force_timeout) {
  const st_layout* L = c.L;
  const int BH = c.B * c.H;
  FwdMaps maps;
  const int el = F16 ? ELEM_F16 : ELEM_BF16;
  if (!make_view_maps(maps.q, q, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.k, k, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.v, v, el, L->geom, BH, c.d))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemFwd) + 1024;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err = cudaSuccess;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    const void* ks[4] = {(const void*)fwd_tc_kernel<F16, false, false>,
                         (const void*)fwd_tc_kernel<F16, true, false>,
                         (const void*)fwd_tc_kernel<F16, false, true>,
                         (const void*)fwd_tc_kernel<F16, true, true>};
    for (int x = 0; x < 4 && err == cudaSuccess; ++x)
      err = cudaFuncSetAttribute(ks[x], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int sms = sm_count();
  const float scale_log2 = c.scale * 1.4426950408889634f;
  const int NH = heads_per_class(c);
  int* slot = L->dev.sched_slots + 2 * (L->next_slot.fetch_add(1) % kSchedSlots);
  record_begin(c);
  for (int pass = 0; pass < L->n_passes; ++pass) {
    const int n = L->dev.n_fwd_items[pass];
    if (n == 0) continue;
    const long long units = (long long)n * NH;
    if (units > 0x7fffffff) return cudaErrorInvalidValue;
    const int grid = (int)std::min<long long>(units, 2LL * sms);
    // the second pass of a two-pass layout merges into the first's O, LSE
    const bool packed = L->geom.cpt > 1;
    auto kernel = pass > 0 ? (packed ? fwd_tc_kernel<F16, true, true> : fwd_tc_kernel<F16, true, false>)
                           : (packed ? fwd_tc_kernel<F16, false, true>
                                     : fwd_tc_kernel<F16, false, false>);
    kernel<<<grid, kThreads, smem, c.stream>>>(
        maps, L->geom, (const FwdItem*)L->dev.fwd_items[pass], (int)units, NH,
        (const KeyEnt*)L->dev.key_ents, heads_of(c), scale_log2, (uint16_t*)o, lse,
        slot, c.status, c.wait_ns, (force_timeout && pass == 0) ? 1 : 0);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  record_end(c);
  return cudaSuccess;
}

}  // namespace

cudaError_t tc_fwd(const Call& c, const void* q, const void* k, const void* v, void* o,
                   float* lse, int force_timeout) {
  return c.dtype == ST_F16 ? tc_fwd_t<true>(c, q, k, v, o, lse, force_timeout)
                           : tc_fwd_t<false>(c, q, k, v, o, lse, force_timeout);
}

}  // namespace st
