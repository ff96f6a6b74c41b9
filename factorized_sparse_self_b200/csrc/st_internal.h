// Internal declarations shared by the host layout builder and the CUDA side
// of libsparse_transformer_attn.so. Not part of the public ABI.
#pragma once

#include <atomic>
#include <cstdint>
#include <vector>

#include "../../include/sparse_transformer_attn.h"

namespace st {

constexpr int kTile = 128;  // query and key tile edge, in view rows
constexpr int kBwdChunk = 8; // most query tiles one backward work item visits
constexpr int kSchedSlots = 64;  // forward calls of one layout that may run at once
// Blocks of the 16-bit backward prologue, each reporting its largest |dout|
// (the backward kernel scales its fp16 copy of dout by a power of two).
constexpr int kDoutSlots = 1024;
// Tail of the 16-bit backward workspace: the backward kernel's work counter
// (first 256 bytes), then kDoutSlots floats.
constexpr size_t kMiscBytes = 256 + 4 * kDoutSlots;

// Row orders ("views") a segment reads its queries or keys in.
enum View : uint8_t {
  VIEW_NAT = 0,  // natural order, position t
  VIEW_SUM = 1,  // summary keys: sigma = floor(j/l)*c + (j mod l) - (l-c)
  VIEW_CLS = 2,  // residue class r = t mod l, row p = floor(t/l); tiles never
                 // straddle classes (each class padded to a multiple of 128)
};

// Membership rule of a segment, in natural coordinates (all imply j <= i).
enum Rule : uint8_t {
  RULE_CAUSAL = 0,          // every j <= i
  RULE_BAND = 1,            // i - l <= j                       (strided A1)
  RULE_BLOCK = 2,           // floor(j/l) == floor(i/l)         (fixed A1)
  RULE_STRIDE = 3,          // (i - j) mod l == 0               (strided A2)
  RULE_STRIDE_FAR = 4,      // (i - j) mod l == 0, i - j >= 2l  (merged strided, beyond band)
  RULE_SUMMARY = 5,         // j mod l >= l - c                 (fixed A2)
  RULE_SUMMARY_EARLIER = 6  // j mod l >= l - c, floor(j/l) < floor(i/l) (merged fixed)
};

enum TileFlag : uint8_t { TILE_FULL = 0, TILE_PARTIAL = 1 };

// ---- device-side schedule records (plain old data, copied as is) ----------

// Forward work item: one query tile of one head class, with its key tiles.
struct FwdItem {
  int32_t qtile;      // tile index in the query view
  int32_t kbeg, kend; // range in the key-entry array
  uint8_t hclass;     // head class (split: 0 even heads, 1 odd heads)
  uint8_t qview;      // View
  uint8_t merge;      // 1: merge with the O/LSE already in the outputs
  uint8_t pad;
};

struct KeyEnt {
  int32_t ktile;  // tile index in the key view
  uint8_t kview;  // View
  uint8_t rule;   // Rule
  uint8_t flag;   // TileFlag
  uint8_t pad;
};

// Backward work item: one key tile of one segment, with its query tiles.
struct BwdItem {
  int32_t ktile;
  int32_t qbeg, qend;  // range in the query-entry array
  uint8_t hclass;
  uint8_t kview;
  uint8_t qview;
  uint8_t rule;
  // How dK, dV of the key tile leave the unit (16-bit path): 0, an fp32
  // reduce-add of the whole tile; 1, a 16-bit store (this unit alone writes
  // every row); 2, a 16-bit store of the whole tile plus an fp32 reduce-add of
  // its summary rows only (a natural key tile of the fixed pattern whose
  // summary keys other units also reach: the epilogue rounds those rows from
  // the accumulator over the stored values).
  uint8_t kv_direct;
  uint8_t pad[3];
};

// Most summary rows of one natural key tile that a kv_direct == 2 unit
// stages: c rows in each of the tile's max(1, 128 / l) l-blocks.
constexpr int kMixedMaxRows = 64;

struct QEnt {
  int32_t qtile;
  uint8_t flag;
  uint8_t q_direct;    // 1: this pair alone produces dQ of its query tile rows
  uint8_t pad[2];
};

// Natural rows of one head class whose gradient needs a given treatment in
// the backward prologue / epilogue (bf16 path).
enum RowList : int {
  ROWS_Q_ACC = 0,   // dQ accumulated in fp32 (several contributions)
  ROWS_K_ACC = 1,   // dK, dV accumulated in fp32
  ROWS_Q_ZERO = 2,  // dQ rows nobody writes: zero-filled
  ROWS_K_ZERO = 3,  // dK, dV rows nobody writes: zero-filled
  N_ROWLISTS = 4
};

// The accumulated rows (ROWS_Q_ACC, ROWS_K_ACC) as segments of consecutive
// rows, at most kSegRows each: the backward prologue zeroes and the epilogue
// rounds one segment per warp, as a contiguous run of memory.
constexpr int kSegRows = 32;
struct RowSeg {
  int32_t start, len;
};

// Heads a call covers: heads h0 .. h0+hn-1 of tensors with B x H heads, for a
// layout with nclasses head classes (kernel parameter, plain old data).
// Division by a divisor that is fixed for a launch, by a multiply-high and a
// shift (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): with s = ceil(log2 d) and m = floor(2^32 (2^s - d)
// / d) + 1, q = (umulhi(m, n) + n) >> s equals floor(n / d) for every
// 0 <= n < 2^31 and 1 <= d < 2^31 (the sum stays below 2^32).
struct FastDiv {
  uint32_t m, s;
};
inline FastDiv make_fastdiv(int32_t d) {
  if (d < 1) d = 1;  // unused divisors (no such view) get a harmless 1
  uint32_t s = 0;
  while ((int64_t(1) << s) < d) ++s;
  const uint64_t m = ((((uint64_t)1 << s) - (uint64_t)d) << 32) / (uint64_t)d + 1;
  return FastDiv{(uint32_t)m, s};
}

struct Heads {
  int32_t B, H, h0, hn, nclasses;
  // head class p (split layouts): its first head index and heads per batch
  // entry among h0 .. h0 + hn - 1
  int32_t first[2], per[2];
  FastDiv fhn, fper[2];
  FastDiv fnh;  // units per work item (heads of the largest class, times B)
};

// Geometry every kernel needs to map view rows to natural positions.
struct Geom {
  int32_t T, l, c;
  int32_t P;       // rows per residue class, T / l (0 when no class view)
  int32_t ptiles;  // 128-row tiles per class, ceil(P / 128)
  // Class-view rows: class r, row p is view row r * cw + p. Short classes
  // (8 <= P <= 64, P dividing 128) are packed, cw = P and cpt = 128 / P whole
  // classes per tile; otherwise each class is padded to cw = 128 * ptiles
  // and cpt = 1.
  int32_t cw, cpt;
  int32_t nsum;    // packed summary rows, (T / l) * c (0 when no summary view)
  int32_t kind, mode;
  int32_t sum_rows;      // summary-view rows of one 128-key tile per l-block, 128 / c
  FastDiv fl, fc, fpt, fcw;  // division by l, c, ptiles and cw
};

// ---- host-side layout ------------------------------------------------------

struct Tile {
  int32_t q, k, live;
  uint8_t flag;
};

struct Segment {
  uint8_t qview, kview, rule;
  int32_t nq, nk;            // tiles in the query / key view
  std::vector<Tile> tiles;   // sorted by (q, k)
};

struct HeadClass {
  std::vector<Segment> segs;
  int64_t nnz = 0;
};

struct DeviceSchedule {
  void* fwd_items[2] = {nullptr, nullptr};  // per forward pass
  int32_t n_fwd_items[2] = {0, 0};
  void* key_ents = nullptr;
  void* bwd_items = nullptr;
  int32_t n_bwd_items = 0;
  // the backward items with every accumulating (not direct) item of two or
  // more query tiles further cut into 2 and into 4 parts; index 0 is bwd_items
  void* bwd_split[3] = {nullptr, nullptr, nullptr};
  int32_t n_bwd_split[3] = {0, 0, 0};
  int32_t max_split_len[3] = {0, 0, 0};  // most query tiles of one item
  int64_t q_ents_total = 0;
  // work counters of the forward kernel: kSchedSlots pairs (next unit, CTAs
  // done), zero between launches (the last CTA of a launch resets its pair)
  int32_t* sched_slots = nullptr;
  void* q_ents = nullptr;
  int32_t max_fwd_keys = 0;    // longest key list of a forward item
  // per head class (at most 2) and row list: device array of natural rows
  void* rows[2][N_ROWLISTS] = {{nullptr, nullptr, nullptr, nullptr},
                               {nullptr, nullptr, nullptr, nullptr}};
  int32_t n_rows[2][N_ROWLISTS] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
  // per head class: segments of ROWS_Q_ACC (index 0) and ROWS_K_ACC (1)
  void* segs[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};
  int32_t n_segs[2][2] = {{0, 0}, {0, 0}};
};

}  // namespace st

struct st_layout {
  st_pattern_desc desc;
  st::Geom geom;
  std::vector<st::HeadClass> hcs;
  int32_t n_passes = 1;      // forward passes (2 for merged strided with class view)
  bool tc_ok = false;        // every segment's rows are intervals (tensor-core path usable)
  bool summary_rows = false; // some backward unit has kv_direct == 2
  // host copies of the schedule
  std::vector<st::FwdItem> fwd_items[2];
  std::vector<st::KeyEnt> key_ents;
  std::vector<st::BwdItem> bwd_items;
  std::vector<st::BwdItem> bwd_split[2];  // parts of 2 and of 4 (see DeviceSchedule)
  std::vector<st::QEnt> q_ents;
  std::vector<int32_t> rows[2][st::N_ROWLISTS];  // see st::RowList
  std::vector<st::RowSeg> segs[2][2];            // see st::RowSeg
  bool on_device = false;
  int device = -1;
  mutable std::atomic<uint32_t> next_slot{0};  // round robin over dev.sched_slots
  st::DeviceSchedule dev;
};

namespace st {
// Implemented in layout.cpp.
st_status build_layout(const st_pattern_desc* desc, st_layout* L);
// Natural-order tiling of the whole set of a head class (export only).
void natural_tiles(const st_layout* L, int hc, std::vector<Tile>& out);
}  // namespace st
