// Host layout builder: pattern -> segments -> 128x128 tiles -> schedule.
//
// "Sparse Transformer" (llm-arch-kb), section 3: the per-query key indices are
// precomputed and attention becomes a block-sparse matmul; section 2 gives
// the two patterns. This builder never materialises a mask or a key list:
// for every query row it writes the live keys of each segment as a few
// intervals in the segment's key view (closed forms of the set definitions),
// and splits those intervals over key tiles to count live pairs per tile.
//
// Segments (disjoint, their union is S_i):
//   dense causal            nat/nat  causal
//   strided split, even h   nat/nat  band            i-l <= j <= i
//   strided split, odd h    cls/cls  stride          p' <= p in class r = i mod l
//   strided merged          nat/nat  band  +  cls/cls stride_far (p' <= p-2)
//   fixed split, even h     nat/nat  block
//   fixed split, odd h      nat/sum  summary         packed summary keys, j <= i
//   fixed merged            nat/nat  block +  nat/sum summary_earlier
// The class view needs T mod l == 0 and l < T, the summary view also c | 128
// and c <= l; without them the same rules run on natural-order keys.
#include <algorithm>
#include <cstring>
#include <utility>

#include "st_internal.h"

namespace st {
namespace {

typedef int64_t i64;

struct SegDef {
  uint8_t qv, kv, rule;
};

bool has_cls(i64 T, i64 l) { return T % l == 0 && l < T; }
bool has_sum(i64 T, i64 l, i64 c) { return has_cls(T, l) && kTile % c == 0 && c <= l; }

std::vector<SegDef> seg_defs(int kind, int mode, int hc, i64 T, i64 l, i64 c) {
  std::vector<SegDef> s;
  if (kind == ST_DENSE_CAUSAL) {
    s.push_back({VIEW_NAT, VIEW_NAT, RULE_CAUSAL});
    return s;
  }
  bool cls = has_cls(T, l), sum = has_sum(T, l, c);
  if (kind == ST_STRIDED) {
    if (mode == ST_HEADS_SPLIT) {
      if (hc == 0)
        s.push_back({VIEW_NAT, VIEW_NAT, RULE_BAND});
      else if (cls)
        s.push_back({VIEW_CLS, VIEW_CLS, RULE_STRIDE});
      else
        s.push_back({VIEW_NAT, VIEW_NAT, RULE_STRIDE});
    } else {
      s.push_back({VIEW_NAT, VIEW_NAT, RULE_BAND});
      if (cls)
        s.push_back({VIEW_CLS, VIEW_CLS, RULE_STRIDE_FAR});
      else
        s.push_back({VIEW_NAT, VIEW_NAT, RULE_STRIDE_FAR});
    }
  } else {
    if (mode == ST_HEADS_SPLIT) {
      if (hc == 0)
        s.push_back({VIEW_NAT, VIEW_NAT, RULE_BLOCK});
      else
        s.push_back({VIEW_NAT, sum ? VIEW_SUM : VIEW_NAT, RULE_SUMMARY});
    } else {
      s.push_back({VIEW_NAT, VIEW_NAT, RULE_BLOCK});
      s.push_back({VIEW_NAT, sum ? VIEW_SUM : VIEW_NAT, RULE_SUMMARY_EARLIER});
    }
  }
  return s;
}

// True when, for every query row, the live keys of this segment form one
// interval of key-view rows (the tensor-core kernels need that).
bool rows_are_intervals(const SegDef& s, i64 T, i64 l) {
  if (s.kv != VIEW_NAT) return true;
  switch (s.rule) {
    case RULE_CAUSAL:
    case RULE_BAND:
    case RULE_BLOCK:
      return true;
    default:
      return l >= T;  // stride / summary rules on natural keys: one run when l >= T
  }
}

i64 view_rows(uint8_t v, const Geom& g) {
  if (v == VIEW_NAT) return g.T;
  if (v == VIEW_SUM) return g.nsum;
  return (i64)g.l * g.cw;  // classes packed or padded to cw rows
}

typedef std::pair<i64, i64> Iv;

// Live keys of query position i (natural) as sorted disjoint half-open
// intervals of key-view rows.
void row_intervals(const SegDef& s, const Geom& g, i64 i, std::vector<Iv>& out) {
  out.clear();
  const i64 l = g.l, c = g.c;
  const i64 W = g.cw;
  auto push = [&](i64 a, i64 b) {
    if (b > a) out.push_back(Iv(a, b));
  };
  switch (s.rule) {
    case RULE_CAUSAL:
      push(0, i + 1);
      break;
    case RULE_BAND:
      push(std::max<i64>(0, i - l), i + 1);
      break;
    case RULE_BLOCK:
      push((i / l) * l, i + 1);
      break;
    case RULE_STRIDE:
    case RULE_STRIDE_FAR: {
      i64 skip = (s.rule == RULE_STRIDE) ? 0 : 2;  // multiples m of l with m >= skip
      if (s.kv == VIEW_CLS) {
        i64 r = i % l, p = i / l;
        push(r * W, r * W + (p - skip + 1));
      } else {
        i64 m_max = i / l;
        for (i64 m = m_max; m >= skip; --m) push(i - m * l, i - m * l + 1);
      }
      break;
    }
    case RULE_SUMMARY:
    case RULE_SUMMARY_EARLIER: {
      i64 blk = i / l, off = i % l;
      if (s.kv == VIEW_SUM) {
        i64 n = blk * c;
        if (s.rule == RULE_SUMMARY) n += std::max<i64>(0, off - (l - c) + 1);
        push(0, n);
      } else {
        i64 last = (s.rule == RULE_SUMMARY) ? blk : blk - 1;
        for (i64 b = 0; b <= last; ++b) push(b * l + (l - c), std::min(b * l + l, i + 1));
      }
      break;
    }
  }
}

// Query positions of a query view, in view-row order: (view row, natural i).
template <class F>
void for_each_query_row(uint8_t qv, const Geom& g, F f) {
  if (qv == VIEW_NAT) {
    for (i64 t = 0; t < g.T; ++t) f(t, t);
  } else {
    const i64 W = g.cw;
    for (i64 r = 0; r < g.l; ++r)
      for (i64 p = 0; p < g.P; ++p) f(r * W + p, p * g.l + r);
  }
}

void build_segment(const SegDef& d, const Geom& g, Segment& seg, int64_t& nnz) {
  seg.qview = d.qv;
  seg.kview = d.kv;
  seg.rule = d.rule;
  seg.nq = (int32_t)((view_rows(d.qv, g) + kTile - 1) / kTile);
  seg.nk = (int32_t)((view_rows(d.kv, g) + kTile - 1) / kTile);
  seg.tiles.clear();
  std::vector<i64> acc((size_t)seg.nk, 0);
  std::vector<int32_t> touched;
  std::vector<Iv> iv;
  i64 cur_q = -1;
  auto flush = [&]() {
    if (cur_q < 0) return;
    std::sort(touched.begin(), touched.end());
    for (int32_t k : touched) {
      Tile t;
      t.q = (int32_t)cur_q;
      t.k = k;
      t.live = (int32_t)acc[(size_t)k];
      t.flag = (t.live == kTile * kTile) ? TILE_FULL : TILE_PARTIAL;
      seg.tiles.push_back(t);
      acc[(size_t)k] = 0;
    }
    touched.clear();
  };
  for_each_query_row(d.qv, g, [&](i64 row, i64 i) {
    i64 qt = row / kTile;
    if (qt != cur_q) {
      flush();
      cur_q = qt;
    }
    row_intervals(d, g, i, iv);
    for (const Iv& x : iv) {
      nnz += x.second - x.first;
      for (i64 kt = x.first / kTile; kt * kTile < x.second; ++kt) {
        i64 a = std::max(x.first, kt * kTile), b = std::min(x.second, (kt + 1) * kTile);
        if (acc[(size_t)kt] == 0) touched.push_back((int32_t)kt);
        acc[(size_t)kt] += b - a;
      }
    }
  });
  flush();
}

// Natural positions of the valid rows of tile `tile` in view v.
void tile_rows(uint8_t v, const Geom& g, int32_t tile, std::vector<int32_t>& out) {
  out.clear();
  for (int k = 0; k < kTile; ++k) {
    if (v == VIEW_NAT) {
      const i64 t = (i64)tile * kTile + k;
      if (t < g.T) out.push_back((int32_t)t);
    } else if (v == VIEW_SUM) {
      const i64 sg = (i64)tile * kTile + k;
      if (sg < g.nsum) out.push_back((int32_t)((sg / g.c) * g.l + (g.l - g.c) + sg % g.c));
    } else {
      const i64 y = (i64)tile * kTile + k, r = y / g.cw, p = y - r * g.cw;
      if (r < g.l && p < g.P) out.push_back((int32_t)(p * g.l + r));
    }
  }
}

// Summary keys of the fixed pattern: the last c positions of each l-block.
bool is_summary_pos(const Geom& g, i64 j) { return j % g.l >= g.l - g.c; }

// A natural key tile whose summary rows form one box of the backward
// kernel's summary-rows tensor map: c rows in each of the tile's
// max(1, 128 / l) l-blocks (l divides 128, or 128 divides l and the tile is
// the last of its block), at most kMixedMaxRows rows.
bool summary_box_fits(const BwdItem& it, const Geom& g) {
  if (it.kview != VIEW_NAT || g.nsum == 0) return false;
  const i64 l = g.l;
  if (l <= kTile) return kTile % l == 0 && g.c * (kTile / l) <= kMixedMaxRows;
  return l % kTile == 0 && ((i64)(it.ktile + 1) * kTile) % l == 0 && g.c <= kMixedMaxRows;
}

// Who writes each gradient row (16-bit path). A backward unit writes dK, dV
// of its whole key tile, a (unit, query tile) pair writes dQ of the query
// tile. A tile whose rows all have exactly one writer is written directly by
// that writer; rows with several writers go through fp32 accumulators; rows
// nobody writes are zero-filled. A natural key tile whose only shared rows are
// summary keys (the fixed pattern's block tiles, whose summary keys later
// query blocks also read) is stored directly and adds its summary rows to the
// accumulators, so that only those rows take the fp32 round trip.
void assign_writers(st_layout* L) {
  const Geom& g = L->geom;
  L->summary_rows = false;
  std::vector<int32_t> rows;
  for (int hc = 0; hc < (int)L->hcs.size(); ++hc) {
    std::vector<int32_t> wk((size_t)g.T, 0), wq((size_t)g.T, 0);
    for (const BwdItem& it : L->bwd_items) {
      if (it.hclass != hc) continue;
      tile_rows(it.kview, g, it.ktile, rows);
      for (int32_t j : rows) wk[(size_t)j] += 1;
      for (int32_t e = it.qbeg; e < it.qend; ++e) {
        tile_rows(it.qview, g, L->q_ents[(size_t)e].qtile, rows);
        for (int32_t i : rows) wq[(size_t)i] += 1;
      }
    }
    std::vector<uint8_t> acck((size_t)g.T, 0), accq((size_t)g.T, 0);
    for (BwdItem& it : L->bwd_items) {
      if (it.hclass != hc) continue;
      tile_rows(it.kview, g, it.ktile, rows);
      bool direct = true;
      for (int32_t j : rows) direct = direct && wk[(size_t)j] == 1;
      uint8_t how = direct ? 1 : 0;
      if (!direct && summary_box_fits(it, g)) {
        bool shared_are_summary = true;
        for (int32_t j : rows)
          shared_are_summary = shared_are_summary && (wk[(size_t)j] == 1 || is_summary_pos(g, j));
        if (shared_are_summary) how = 2;
      }
      it.kv_direct = how;
      if (how == 2) L->summary_rows = true;
      // every summary row of a kv_direct == 2 tile is reduce-added (the box
      // covers them all), so all of them are accumulated and rounded
      for (int32_t j : rows)
        if (how == 0 || (how == 2 && is_summary_pos(g, j))) acck[(size_t)j] = 1;
      for (int32_t e = it.qbeg; e < it.qend; ++e) {
        QEnt& qe = L->q_ents[(size_t)e];
        tile_rows(it.qview, g, qe.qtile, rows);
        bool qd = true;
        for (int32_t i : rows) qd = qd && wq[(size_t)i] == 1;
        qe.q_direct = qd ? 1 : 0;
        if (!qd)
          for (int32_t i : rows) accq[(size_t)i] = 1;
      }
    }
    for (int k = 0; k < N_ROWLISTS; ++k) L->rows[hc][k].clear();
    for (int32_t t = 0; t < g.T; ++t) {
      if (accq[(size_t)t]) L->rows[hc][ROWS_Q_ACC].push_back(t);
      if (acck[(size_t)t]) L->rows[hc][ROWS_K_ACC].push_back(t);
      if (wq[(size_t)t] == 0) L->rows[hc][ROWS_Q_ZERO].push_back(t);
      if (wk[(size_t)t] == 0) L->rows[hc][ROWS_K_ZERO].push_back(t);
    }
    // the accumulated rows as runs of consecutive rows, cut at kSegRows
    for (int k = 0; k < 2; ++k) {
      const std::vector<int32_t>& rl = L->rows[hc][k ? ROWS_K_ACC : ROWS_Q_ACC];
      std::vector<RowSeg>& sg = L->segs[hc][k];
      sg.clear();
      for (size_t a = 0; a < rl.size();) {
        size_t b = a + 1;
        while (b < rl.size() && rl[b] == rl[b - 1] + 1 && (int)(b - a) < kSegRows) ++b;
        sg.push_back(RowSeg{rl[a], (int32_t)(b - a)});
        a = b;
      }
    }
  }
}

}  // namespace

st_status build_layout(const st_pattern_desc* desc, st_layout* L) {
  const i64 T = desc->T, l = desc->l;
  i64 c = desc->c;
  if (T < 1 || T > (1 << 30)) return ST_ERR_INVALID;
  if (desc->kind < ST_STRIDED || desc->kind > ST_DENSE_CAUSAL) return ST_ERR_INVALID;
  int mode = desc->head_mode;
  if (desc->kind == ST_DENSE_CAUSAL) {
    mode = ST_HEADS_MERGED;
  } else {
    if (mode != ST_HEADS_SPLIT && mode != ST_HEADS_MERGED) return ST_ERR_INVALID;
    if (l < 1) return ST_ERR_INVALID;
  }
  if (desc->kind == ST_FIXED) {
    if (c < 1 || c > l) return ST_ERR_INVALID;
  } else {
    c = 1;
  }
  L->desc = *desc;
  L->desc.head_mode = mode;
  L->desc.c = (int32_t)c;
  if (desc->kind == ST_DENSE_CAUSAL) L->desc.l = (int32_t)std::max<i64>(l, 1);
  Geom& g = L->geom;
  std::memset(&g, 0, sizeof(g));
  g.T = (int32_t)T;
  g.l = L->desc.l;
  g.c = (int32_t)c;
  g.kind = desc->kind;
  g.mode = mode;
  if (desc->kind != ST_DENSE_CAUSAL && has_cls(T, g.l)) {
    g.P = (int32_t)(T / g.l);
    g.ptiles = (g.P + kTile - 1) / kTile;
    // (only the strided pattern uses the class view; the others keep cpt = 1
    // so that their launches take the kernels without the packed paths)
    const bool packed =
        desc->kind == ST_STRIDED && g.P >= 8 && g.P <= 64 && kTile % g.P == 0;
    g.cw = packed ? g.P : g.ptiles * kTile;
    g.cpt = packed ? kTile / g.P : 1;
  }
  if (desc->kind == ST_FIXED && has_sum(T, g.l, c)) g.nsum = (int32_t)((T / g.l) * c);
  g.sum_rows = g.c >= 1 ? kTile / g.c : 0;
  g.fl = make_fastdiv(g.l);
  g.fc = make_fastdiv(g.c);
  g.fpt = make_fastdiv(g.ptiles);
  g.fcw = make_fastdiv(g.cw);

  int nhc = (desc->kind != ST_DENSE_CAUSAL && mode == ST_HEADS_SPLIT) ? 2 : 1;
  L->hcs.assign((size_t)nhc, HeadClass());
  L->tc_ok = true;
  for (int hc = 0; hc < nhc; ++hc) {
    std::vector<SegDef> defs = seg_defs(desc->kind, mode, hc, T, g.l, c);
    HeadClass& H = L->hcs[(size_t)hc];
    H.segs.resize(defs.size());
    H.nnz = 0;
    for (size_t s = 0; s < defs.size(); ++s) {
      build_segment(defs[s], g, H.segs[s], H.nnz);
      if (!rows_are_intervals(defs[s], T, g.l)) L->tc_ok = false;
    }
  }

  // ---- forward schedule: passes group the segments by query view ----------
  L->n_passes = 1;
  for (int p = 0; p < 2; ++p) L->fwd_items[p].clear();
  L->key_ents.clear();
  struct Pending {
    FwdItem it;
    std::vector<KeyEnt> keys;
  };
  for (int pass = 0; pass < 2; ++pass) {
    std::vector<Pending> items;
    for (int hc = 0; hc < nhc; ++hc) {
      const HeadClass& H = L->hcs[(size_t)hc];
      uint8_t qv0 = H.segs[0].qview;
      std::vector<const Segment*> group;
      for (const Segment& s : H.segs)
        if ((pass == 0) == (s.qview == qv0)) group.push_back(&s);
      if (group.empty()) continue;
      if (pass == 1) L->n_passes = 2;
      int32_t nq = group[0]->nq;
      std::vector<Pending> per_q((size_t)nq);
      for (int32_t q = 0; q < nq; ++q) {
        per_q[(size_t)q].it.qtile = q;
        per_q[(size_t)q].it.hclass = (uint8_t)hc;
        per_q[(size_t)q].it.qview = group[0]->qview;
        per_q[(size_t)q].it.merge = (uint8_t)pass;
        per_q[(size_t)q].it.pad = 0;
      }
      for (const Segment* s : group)
        for (const Tile& t : s->tiles) {
          KeyEnt e;
          e.ktile = t.k;
          e.kview = s->kview;
          e.rule = s->rule;
          e.flag = t.flag;
          e.pad = 0;
          per_q[(size_t)t.q].keys.push_back(e);
        }
      for (Pending& p : per_q)
        if (pass == 0 || !p.keys.empty()) items.push_back(std::move(p));
    }
    if (pass == 1 && items.empty()) break;
    // longest key lists first (stable: ties keep head class, tile order)
    std::stable_sort(items.begin(), items.end(), [](const Pending& a, const Pending& b) {
      return a.keys.size() > b.keys.size();
    });
    for (Pending& p : items) {
      p.it.kbeg = (int32_t)L->key_ents.size();
      L->key_ents.insert(L->key_ents.end(), p.keys.begin(), p.keys.end());
      p.it.kend = (int32_t)L->key_ents.size();
      L->fwd_items[pass].push_back(p.it);
    }
  }

  // ---- backward schedule: key-major over every segment ---------------------
  L->bwd_items.clear();
  L->q_ents.clear();
  struct PendingB {
    BwdItem it;
    std::vector<QEnt> qs;
  };
  std::vector<PendingB> bitems;
  for (int hc = 0; hc < nhc; ++hc) {
    const HeadClass& H = L->hcs[(size_t)hc];
    for (const Segment& s : H.segs) {
      std::vector<PendingB> per_k((size_t)s.nk);
      for (const Tile& t : s.tiles) {
        QEnt e;
        e.qtile = t.q;
        e.flag = t.flag;
        e.q_direct = 0;
        e.pad[0] = e.pad[1] = 0;
        per_k[(size_t)t.k].qs.push_back(e);
      }
      for (int32_t k = 0; k < s.nk; ++k) {
        PendingB& p = per_k[(size_t)k];
        if (p.qs.empty()) continue;
        p.it.ktile = k;
        p.it.hclass = (uint8_t)hc;
        p.it.kview = s.kview;
        p.it.qview = s.qview;
        p.it.rule = s.rule;
        // Long key columns (summary keys are read by every later query tile)
        // are cut into chunks so that no CTA carries a whole column; each
        // chunk reduce-adds its own dK, dV partial.
        const size_t nq = p.qs.size();
        const size_t nchunks = (nq + kBwdChunk - 1) / kBwdChunk;
        for (size_t ch = 0; ch < nchunks; ++ch) {
          const size_t a = nq * ch / nchunks, b = nq * (ch + 1) / nchunks;
          PendingB part;
          part.it = p.it;
          part.qs.assign(p.qs.begin() + a, p.qs.begin() + b);
          bitems.push_back(std::move(part));
        }
      }
    }
  }
  std::stable_sort(bitems.begin(), bitems.end(), [](const PendingB& a, const PendingB& b) {
    return a.qs.size() > b.qs.size();
  });
  for (PendingB& p : bitems) {
    p.it.qbeg = (int32_t)L->q_ents.size();
    L->q_ents.insert(L->q_ents.end(), p.qs.begin(), p.qs.end());
    p.it.qend = (int32_t)L->q_ents.size();
    p.it.kv_direct = 0;
    p.it.pad[0] = p.it.pad[1] = p.it.pad[2] = 0;
    L->bwd_items.push_back(p.it);
  }
  assign_writers(L);
  // Finer cuts of the accumulating items, for launches with few units per
  // CTA: a key tile that already has several writers may take more (each part
  // reduce-adds its dK, dV partial); direct items stay whole.
  for (int f = 0; f < 2; ++f) {
    const int32_t parts = f == 0 ? 2 : 4;
    std::vector<BwdItem>& out = L->bwd_split[f];
    out.clear();
    for (const BwdItem& it : L->bwd_items) {
      const int32_t nq = it.qend - it.qbeg;
      const int32_t np = (it.kv_direct || nq < 2) ? 1 : std::min(parts, nq);
      for (int32_t x = 0; x < np; ++x) {
        BwdItem part = it;
        part.qbeg = it.qbeg + (int32_t)((int64_t)nq * x / np);
        part.qend = it.qbeg + (int32_t)((int64_t)nq * (x + 1) / np);
        out.push_back(part);
      }
    }
    std::stable_sort(out.begin(), out.end(), [](const BwdItem& a, const BwdItem& b) {
      return a.qend - a.qbeg > b.qend - b.qbeg;
    });
  }
  return ST_OK;
}

void natural_tiles(const st_layout* L, int hc, std::vector<Tile>& out) {
  const Geom& g = L->geom;
  const HeadClass& H = L->hcs[(size_t)hc];
  const i64 nt = (g.T + kTile - 1) / kTile;
  const i64 W = g.cw;
  out.clear();
  std::vector<i64> acc((size_t)nt, 0);
  std::vector<int32_t> touched;
  std::vector<Iv> iv;
  std::vector<SegDef> defs;
  for (const Segment& s : H.segs) defs.push_back({s.qview, s.kview, s.rule});
  for (i64 qt = 0; qt < nt; ++qt) {
    for (i64 i = qt * kTile; i < std::min<i64>(g.T, (qt + 1) * kTile); ++i) {
      for (const SegDef& d : defs) {
        row_intervals(d, g, i, iv);
        for (const Iv& x : iv) {
          if (d.kv == VIEW_NAT) {
            for (i64 kt = x.first / kTile; kt * kTile < x.second; ++kt) {
              i64 a = std::max(x.first, kt * kTile), b = std::min(x.second, (kt + 1) * kTile);
              if (acc[(size_t)kt] == 0) touched.push_back((int32_t)kt);
              acc[(size_t)kt] += b - a;
            }
          } else {
            for (i64 y = x.first; y < x.second; ++y) {
              i64 j;
              if (d.kv == VIEW_SUM)
                j = (y / g.c) * g.l + (g.l - g.c) + y % g.c;
              else
                j = (y % W) * g.l + y / W;
              i64 kt = j / kTile;
              if (acc[(size_t)kt] == 0) touched.push_back((int32_t)kt);
              acc[(size_t)kt] += 1;
            }
          }
        }
      }
    }
    std::sort(touched.begin(), touched.end());
    for (int32_t k : touched) {
      Tile t;
      t.q = (int32_t)qt;
      t.k = k;
      t.live = (int32_t)acc[(size_t)k];
      t.flag = (t.live == kTile * kTile) ? TILE_FULL : TILE_PARTIAL;
      out.push_back(t);
      acc[(size_t)k] = 0;
    }
    touched.clear();
  }
}

}  // namespace st
