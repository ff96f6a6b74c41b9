// Forward pass on the tensor cores (sm_100a): tcgen05.mma with TMEM
// accumulators, TMA-staged tiles, online softmax.
//
// Computes O_i = softmax(scale q_i K_{S_i}^T) V_{S_i} and LSE_i over the live
// tiles of each query tile ("Sparse Transformer", llm-arch-kb, section 2,
// "Per-layer cost": a block-sparse matmul over the pattern's blocks; the
// milestone page, "The notation", for the attention itself).
//
// One CTA = one query tile (128 rows of one head, in its segment's row order)
// and its key tiles. Warp roles:
//   warp 0       TMA producer: the Q tile once, then K and V tiles into a
//                3-stage ring (natural, summary or residue-class view);
//   warp 1       TMEM owner and MMA issuer: S = Q K^T (M=128, N=128, K=64)
//                into one of two TMEM S buffers, then O += P V (M=128, N=64,
//                K=128) into the TMEM O accumulator;
//   warps 2..5   softmax: thread = query row = TMEM lane. Loads S, applies the
//                row's live-key interval on PARTIAL tiles, keeps the running
//                max (rescaling O in TMEM only when the max grows by more
//                than 2^8) and the running sum, writes P as bf16 into a
//                128B-swizzled shared tile for the PV MMA; at the end
//                normalises O, merges with a previous pass if asked, and
//                stores O (TMA) and LSE.
// Every wait is bounded; a wait that runs out sets the status word, raises
// the CTA's abort flag, and all roles drain their in-flight work and return.
#include <math.h>

#include "launch.h"
#include "tc_common.cuh"

namespace st {
namespace {

using namespace tc;

constexpr int NS = 3;                     // K/V stages
constexpr int kTileBytes = kTile * 64 * 2;  // one 128 x 64 bf16 tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdMaps {
  CUtensorMap q[3], k[3], v[3], o[3];  // indexed by View
};

struct SmemFwd {
  uint8_t q[kTileBytes];          // Q tile; later stages the O tile for the store
  uint8_t k[NS][kTileBytes];
  uint8_t v[NS][kTileBytes];
  uint8_t p[2][2 * kTileBytes];   // P tiles: keys 0-63 and 64-127 as two K-blocks
  uint8_t oprev[kTileBytes];      // merge pass: O of the previous pass
  uint64_t q_full, oprev_full, o_done, stage_done, fin;
  uint64_t kv_full[NS], kv_empty[NS], s_full[2], p_full[2];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void load_tile(void* dst, const CUtensorMap* maps, int view,
                                          const Geom& g, int tile, int bh, uint64_t* bar) {
  if (view == VIEW_NAT) {
    tma_load_3d(dst, &maps[VIEW_NAT], bar, 0, tile * kTile, bh);
  } else if (view == VIEW_SUM) {
    tma_load_4d(dst, &maps[VIEW_SUM], bar, 0, g.l - g.c, tile * (kTile / g.c), bh);
  } else {
    int r = tile / g.ptiles, pb = tile - r * g.ptiles;
    tma_load_4d(dst, &maps[VIEW_CLS], bar, 0, r, pb * kTile, bh);
  }
}

__device__ __forceinline__ void store_tile(const CUtensorMap* maps, int view, const Geom& g,
                                           int tile, int bh, const void* src) {
  if (view == VIEW_NAT) {
    tma_store_3d(&maps[VIEW_NAT], src, 0, tile * kTile, bh);
  } else {
    int r = tile / g.ptiles, pb = tile - r * g.ptiles;
    tma_store_4d(&maps[VIEW_CLS], src, 0, r, pb * kTile, bh);
  }
}

// Live key columns [lo, hi) of key tile `ke` for the query at natural
// position i (and, in the residue view, its class row p = i / l). The bounds
// restate the segment rules as intervals.
__device__ __forceinline__ void live_cols(const Geom& g, const KeyEnt& ke, int i, int& lo,
                                          int& hi) {
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
      case RULE_BLOCK: a = (i / l) * l; b = i + 1; break;
      case RULE_STRIDE: a = i; b = i + 1; break;          // natural keys only when l >= T
      case RULE_SUMMARY: a = l - c; b = i + 1; break;     // natural keys only when l >= T
      default: a = 0; b = 0; break;                        // stride_far / summary_earlier: empty
    }
  } else if (ke.kview == VIEW_SUM) {
    base = ke.ktile * kTile;
    lim = g.nsum;
    const int blk = i / l, off = i - blk * l;
    a = 0;
    b = blk * c + ((ke.rule == RULE_SUMMARY) ? max(0, off - (l - c) + 1) : 0);
  } else {
    const int pb = ke.ktile % g.ptiles;
    base = pb * kTile;
    lim = g.P;
    const int p = i / l;
    a = 0;
    b = (ke.rule == RULE_STRIDE) ? p + 1 : p - 1;
  }
  b = min(b, lim);
  lo = max(a - base, 0);
  hi = min(b - base, kTile);
  if (hi < lo) hi = lo;
}

__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ FwdMaps maps, Geom g, const FwdItem* __restrict__ items,
              const KeyEnt* __restrict__ keys, int B, int H, int nclasses, float scale_log2,
              float* __restrict__ lse, int* status, uint64_t wait_ns, int force_timeout) {
  extern __shared__ uint8_t smem_raw[];
  SmemFwd& S = *reinterpret_cast<SmemFwd*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const FwdItem it = items[blockIdx.y];
  const int bh = head_of(blockIdx.x, it.hclass, B, H, nclasses);
  if (bh < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = it.kend - it.kbeg;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    mbar_init(&S.q_full, 1);
    mbar_init(&S.oprev_full, 1);
    mbar_init(&S.o_done, 1);
    mbar_init(&S.stage_done, 128);
    mbar_init(&S.fin, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.s_full[b], 1);
      mbar_init(&S.p_full[b], 128);
    }
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  auto fail = [&]() {
    *abort = 1;
    set_status(status, ST_ERR_DEVICE_TIMEOUT);
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued[NS];
      for (int s = 0; s < NS; ++s) issued[s] = -1;
      mbar_arrive_expect_tx(&S.q_full, kTileBytes);
      load_tile(S.q, maps.q, it.qview, g, it.qtile, bh, &S.q_full);
      if (it.merge) {
        mbar_arrive_expect_tx(&S.oprev_full, kTileBytes);
        load_tile(S.oprev, maps.o, it.qview, g, it.qtile, bh, &S.oprev_full);
      }
      for (int e = 0; e < n; ++e) {
        const int s = e % NS;
        if (e >= NS && !mbar_wait(&S.kv_empty[s], ((e / NS) - 1) & 1, wait_ns, abort)) {
          fail();
          break;
        }
        if (force_timeout && e == 0) continue;  // test hook: this stage never fills
        const KeyEnt ke = keys[it.kbeg + e];
        mbar_arrive_expect_tx(&S.kv_full[s], 2 * kTileBytes);
        load_tile(S.k[s], maps.k, ke.kview, g, ke.ktile, bh, &S.kv_full[s]);
        load_tile(S.v[s], maps.v, ke.kview, g, ke.ktile, bh, &S.kv_full[s]);
        issued[s] = e;
      }
      // no copy may be in flight when the CTA exits
      mbar_wait(&S.q_full, 0, wait_ns, abort);
      if (it.merge) mbar_wait(&S.oprev_full, 0, wait_ns, abort);
      for (int s = 0; s < NS; ++s)
        if (issued[s] >= 0 && !mbar_wait(&S.kv_full[s], (issued[s] / NS) & 1, wait_ns, abort))
          fail();
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idPV = idesc_bf16(128, 64, false, true);
      const uint32_t q_addr = smem_u32(S.q);
      bool ok = mbar_wait(&S.q_full, 0, wait_ns, abort);
      auto issue_s = [&](int e) -> bool {
        const int s = e % NS, b = e & 1;
        if (!mbar_wait(&S.kv_full[s], (e / NS) & 1, wait_ns, abort)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(S.k[s]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + b * 128, sdesc(q_addr + kk * 32, 16, 1024),
                 sdesc(k_addr + kk * 32, 16, 1024), idS, kk > 0);
        mma_commit(&S.s_full[b]);
        return true;
      };
      if (ok && n > 0) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int e = 0; ok && e < n; ++e) {
        const int s = e % NS, b = e & 1;
        if (!mbar_wait(&S.p_full[b], (e >> 1) & 1, wait_ns, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t p_addr = smem_u32(S.p[b]);
        const uint32_t v_addr = smem_u32(S.v[s]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + kColO, sdesc(p_addr + (kk >> 2) * kTileBytes + (kk & 3) * 32, 16, 1024),
                 sdesc(v_addr + kk * 2048, 16384, 1024), idPV, (e > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&S.o_done);
        mma_commit(&S.kv_empty[s]);
        if (e + 2 < n) ok = issue_s(e + 2);
      }
      if (!ok) fail();
      mma_commit(&S.fin);
      mbar_wait(&S.fin, 0, wait_ns, abort);
    }
  } else {
    // ---------------- softmax warps ----------------
    const int lg = warp & 3;                 // TMEM lane group of this warp
    const int row = lg * 32 + lane;          // query row in the tile = TMEM lane
    const uint32_t tl = (uint32_t)(lg * 32) << 16;
    const int i = view_pos(g, it.qview, it.qtile, row);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int e = 0; e < n; ++e) {
      const int b = e & 1;
      const KeyEnt ke = keys[it.kbeg + e];
      ok = mbar_wait(&S.s_full[b], (e >> 1) & 1, wait_ns, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        tmem_ld32(tmem + tl + b * 128 + c4 * 32, reinterpret_cast<uint32_t*>(s) + c4 * 32);
      tmem_wait_ld();
      if (ke.flag != TILE_FULL) {
        int lo, hi;
        live_cols(g, ke, i, lo, hi);
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (x < lo || x >= hi) s[x] = -INFINITY;
      }
      float mt = s[0];
#pragma unroll
      for (int x = 1; x < 128; ++x) mt = fmaxf(mt, s[x]);
      mt *= scale_log2;
      const float m_new = fmaxf(m_run, mt);
      float alpha = 1.f;
      bool rescale_o = false;
      if (m_new > m_run + kRescaleThreshold) {
        rescale_o = (m_run != -INFINITY);
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
      }
      const float mu = (m_run == -INFINITY) ? 0.f : m_run;
      float rs = 0.f;
      const uint32_t pb = smem_u32(S.p[b]);
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        float p8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          p8[x] = fast_exp2(fmaf(s[ch * 8 + x], scale_log2, -mu));
          rs += p8[x];
        }
        st_shared_v4(pb + (ch >> 3) * kTileBytes + swz128(row, ch & 7), pack_bf16(p8[0], p8[1]),
                     pack_bf16(p8[2], p8[3]), pack_bf16(p8[4], p8[5]), pack_bf16(p8[6], p8[7]));
      }
      l_run = l_run * alpha + rs;
      if (e > 0) {
        ok = mbar_wait(&S.o_done, (e - 1) & 1, wait_ns, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale_o)) {
          const float a = rescale_o ? alpha : 1.f;
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            uint32_t o[32];
            tmem_ld32(tmem + tl + kColO + c2 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * a);
            tmem_st32(tmem + tl + kColO + c2 * 32, o);
          }
          tmem_wait_st();
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&S.p_full[b]);
    }
    if (!ok) {
      fail();
    } else {
      // ---- epilogue ----
      float out[64];
      if (n > 0) {
        ok = mbar_wait(&S.o_done, (n - 1) & 1, wait_ns, abort);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok && it.merge) ok = __all_sync(0xffffffffu, mbar_wait(&S.oprev_full, 0, wait_ns, abort));
      if (!ok) {
        fail();
      } else {
        if (n > 0) {
          tc_fence_after();
          tmem_ld32(tmem + tl + kColO, reinterpret_cast<uint32_t*>(out));
          tmem_ld32(tmem + tl + kColO + 32, reinterpret_cast<uint32_t*>(out) + 32);
          tmem_wait_ld();
        }
        const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
        float L = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
#pragma unroll
        for (int x = 0; x < 64; ++x) out[x] = (n > 0) ? out[x] * inv : 0.f;
        if (it.merge && i >= 0) {
          const float Lp = lse[(size_t)bh * g.T + i];
          const float mx = fmaxf(Lp, L);
          float wp = 0.f, wc = 0.f;
          if (mx != -INFINITY) {
            const float Ln = mx + __logf(__expf(Lp - mx) + __expf(L - mx));
            wp = __expf(Lp - Ln);
            wc = __expf(L - Ln);
            L = Ln;
          }
          const uint32_t ob = smem_u32(S.oprev);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t w[4];
            ld_shared_v4(ob + swz128(row, ch), w[0], w[1], w[2], w[3]);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w[x]);
              float2 f = __bfloat1622float2(h);
              out[ch * 8 + 2 * x] = fmaf(wp, f.x, wc * out[ch * 8 + 2 * x]);
              out[ch * 8 + 2 * x + 1] = fmaf(wp, f.y, wc * out[ch * 8 + 2 * x + 1]);
            }
          }
        }
        const uint32_t qb = smem_u32(S.q);  // Q is no longer read: stage O here
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(qb + swz128(row, ch), pack_bf16(out[ch * 8 + 0], out[ch * 8 + 1]),
                       pack_bf16(out[ch * 8 + 2], out[ch * 8 + 3]),
                       pack_bf16(out[ch * 8 + 4], out[ch * 8 + 5]),
                       pack_bf16(out[ch * 8 + 6], out[ch * 8 + 7]));
        if (i >= 0) lse[(size_t)bh * g.T + i] = L;
        fence_async_smem();
        mbar_arrive(&S.stage_done);
        if (warp == 2 && lane == 0) {
          if (mbar_wait(&S.stage_done, 0, wait_ns, abort)) {
            store_tile(maps.o, it.qview, g, it.qtile, bh, S.q);
            bulk_commit();
            bulk_wait_all();
          } else {
            fail();
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace
}  // namespace st

namespace st {

cudaError_t tc_fwd(const Call& c, const void* q, const void* k, const void* v, void* o,
                   float* lse, int force_timeout) {
  const st_layout* L = c.L;
  const int BH = c.B * c.H;
  FwdMaps maps;
  if (!make_view_maps(maps.q, q, false, L->geom, BH, c.d) ||
      !make_view_maps(maps.k, k, false, L->geom, BH, c.d) ||
      !make_view_maps(maps.v, v, false, L->geom, BH, c.d) ||
      !make_view_maps(maps.o, o, false, L->geom, BH, c.d))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemFwd) + 1024;
  cudaError_t err =
      cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const float scale_log2 = c.scale * 1.4426950408889634f;
  for (int pass = 0; pass < L->n_passes; ++pass) {
    const int n = L->dev.n_fwd_items[pass];
    if (n == 0) continue;
    dim3 grid(heads_per_class(c), n);
    fwd_tc_kernel<<<grid, kThreads, smem, c.stream>>>(
        maps, L->geom, (const FwdItem*)L->dev.fwd_items[pass], (const KeyEnt*)L->dev.key_ents,
        c.B, c.H, c.nclasses, scale_log2, lse, c.status, c.wait_ns,
        (force_timeout && pass == 0) ? 1 : 0);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace st
