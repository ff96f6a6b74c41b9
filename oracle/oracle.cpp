// Plain CPU oracle for factorized causal self-attention (Sparse Transformer).
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this code:
// only the test suite, the smoke check and the CPU-baseline leg of the
// benchmark load it. It shares no source, header or table with the CUDA
// library; it reads inputs as float32 (bf16 values widen to float exactly)
// and does every step in double precision.
//
// What it follows:
//  * Index sets: "Sparse Transformer" (llm-arch-kb), section 2 Derivation,
//    "Pattern A - strided" (local window plus every l-th earlier key) and
//    "Pattern B - fixed" (own l-block plus the summary positions of each
//    block); nlp-lineage "Sparse Transformer" milestone, "The idea" (the two
//    factors, each split between two heads; summaries at the end of a block).
//    Readings used where the extracted set-builder formulas are missing:
//      strided A1_i = { j : max(0, i-l) <= j <= i }
//      strided A2_i = { j : 0 <= j <= i, (i-j) mod l == 0 }
//      fixed   A1_i = { j <= i : floor(j/l) == floor(i/l) }
//      fixed   A2_i = { j <= i : j mod l >= l - c }   (last c of each block)
//      dense causal S_i = { j <= i }
//    split heads: head h uses A1 when h is even, A2 when h is odd;
//    merged heads: S_i = A1_i union A2_i.
//  * Attention over an allowed set: nlp-lineage milestone, "The notation":
//    softmax(q_i K_{S_i}^T / sqrt(d)) V_{S_i}; llm-arch-kb section 2,
//    "Sparse attention as an unnormalized form": the softmax normalises over
//    S_i only. An empty S_i gives O_i = 0, LSE_i = -inf and no gradient.
//  * Backward with recomputation: nlp-lineage milestone, "The idea"
//    (attention weights recomputed when the gradients need them): P is
//    rebuilt from the inputs, never stored.
//
// parity pins: see tests/test_oracle_pins.py (closed-form row counts, dense
// masked attention via a library routine, finite differences, special
// cases l >= T and Q = 0, exact gradient invariants).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum Kind { STRIDED = 0, FIXED = 1, DENSE_CAUSAL = 2 };
enum Mode { SPLIT = 0, MERGED = 1 };

typedef int64_t i64;

// ---- explicit index sets -------------------------------------------------

// Append the strided local window A1_i.
void strided_a1(i64 i, i64 l, std::vector<i64>& out) {
  i64 lo = i - l;
  if (lo < 0) lo = 0;
  for (i64 j = lo; j <= i; ++j) out.push_back(j);
}

// Append the strided long-range set A2_i: i, i-l, i-2l, ... >= 0.
void strided_a2(i64 i, i64 l, std::vector<i64>& out) {
  for (i64 j = i; j >= 0; j -= l) out.push_back(j);
}

// Append the fixed own-block set A1_i.
void fixed_a1(i64 i, i64 l, std::vector<i64>& out) {
  for (i64 j = (i / l) * l; j <= i; ++j) out.push_back(j);
}

// Append the fixed summary set A2_i: in every block b <= floor(i/l), the
// positions b*l + (l-c) .. b*l + l-1 that are <= i.
void fixed_a2(i64 i, i64 l, i64 c, std::vector<i64>& out) {
  for (i64 b = 0; b <= i / l; ++b) {
    for (i64 off = l - c; off < l; ++off) {
      i64 j = b * l + off;
      if (j >= 0 && j <= i) out.push_back(j);
    }
  }
}

// The sorted, duplicate-free set S_{h,i}.
void row_set(int kind, int mode, i64 l, i64 c, i64 h, i64 i, std::vector<i64>& s) {
  s.clear();
  if (kind == DENSE_CAUSAL) {
    for (i64 j = 0; j <= i; ++j) s.push_back(j);
    return;
  }
  bool use1 = (mode == MERGED) || (h % 2 == 0);
  bool use2 = (mode == MERGED) || (h % 2 == 1);
  if (kind == STRIDED) {
    if (use1) strided_a1(i, l, s);
    if (use2) strided_a2(i, l, s);
  } else {
    if (use1) fixed_a1(i, l, s);
    if (use2) fixed_a2(i, l, c, s);
  }
  std::sort(s.begin(), s.end());
  s.erase(std::unique(s.begin(), s.end()), s.end());
}

bool row_has(const std::vector<i64>& s, i64 j) {
  return std::binary_search(s.begin(), s.end(), j);
}

// ---- attention arithmetic, one query row ---------------------------------

struct Dims {
  i64 B, H, T, d;
};

inline const float* rowp(const float* x, const Dims& D, i64 bh, i64 t) {
  return x + (bh * D.T + t) * D.d;
}

double dot(const float* a, const float* b, i64 d) {
  double acc = 0.0;
  for (i64 k = 0; k < d; ++k) acc += (double)a[k] * (double)b[k];
  return acc;
}

// Softmax of one row over its set: fills p (probabilities) and returns LSE.
// Empty set: returns -inf and leaves p empty.
double row_softmax(const float* q, const float* k, const Dims& D, i64 bh, double scale,
                   const std::vector<i64>& s, std::vector<double>& p) {
  p.assign(s.size(), 0.0);
  if (s.empty()) return -std::numeric_limits<double>::infinity();
  double m = -std::numeric_limits<double>::infinity();
  for (size_t t = 0; t < s.size(); ++t) {
    p[t] = scale * dot(q, rowp(k, D, bh, s[t]), D.d);
    if (p[t] > m) m = p[t];
  }
  double z = 0.0;
  for (size_t t = 0; t < s.size(); ++t) {
    p[t] = std::exp(p[t] - m);
    z += p[t];
  }
  for (size_t t = 0; t < s.size(); ++t) p[t] /= z;
  return m + std::log(z);
}

void set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

}  // namespace

extern "C" {

// Number of OpenMP threads the oracle will use.
int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Writes the sorted set S_{h,i} into out (at most cap entries); returns |S_{h,i}|.
i64 orc_row_set(int kind, int mode, i64 l, i64 c, i64 h, i64 i, i64* out, i64 cap) {
  std::vector<i64> s;
  row_set(kind, mode, l, c, h, i, s);
  for (i64 t = 0; t < (i64)s.size() && t < cap; ++t) out[t] = s[t];
  return (i64)s.size();
}

// Total number of live (i, j) pairs of head h over a length-T sequence.
i64 orc_nnz(int kind, int mode, i64 T, i64 l, i64 c, i64 h) {
  std::vector<i64> s;
  i64 n = 0;
  for (i64 i = 0; i < T; ++i) {
    row_set(kind, mode, l, c, h, i, s);
    n += (i64)s.size();
  }
  return n;
}

// Forward over all (b, h, i). q, k, v: [B,H,T,d] float; o: [B,H,T,d] double;
// lse: [B,H,T] double (natural log).
void orc_forward(int kind, int mode, i64 B, i64 H, i64 T, i64 d, i64 l, i64 c, double scale,
                 const float* q, const float* k, const float* v, double* o, double* lse,
                 int nthreads) {
  Dims D{B, H, T, d};
  set_threads(nthreads);
#pragma omp parallel
  {
    std::vector<i64> s;
    std::vector<double> p;
#pragma omp for schedule(dynamic, 16) collapse(2)
    for (i64 bh = 0; bh < B * H; ++bh) {
      for (i64 i = 0; i < T; ++i) {
        i64 h = bh % H;
        row_set(kind, mode, l, c, h, i, s);
        double L = row_softmax(rowp(q, D, bh, i), k, D, bh, scale, s, p);
        double* oi = o + (bh * T + i) * d;
        for (i64 x = 0; x < d; ++x) oi[x] = 0.0;
        for (size_t t = 0; t < s.size(); ++t) {
          const float* vj = rowp(v, D, bh, s[t]);
          for (i64 x = 0; x < d; ++x) oi[x] += p[t] * (double)vj[x];
        }
        lse[bh * T + i] = L;
      }
    }
  }
}

// Forward for selected rows only: row r is (bh[r], i[r]); o: [n, d], lse: [n].
void orc_forward_rows(int kind, int mode, i64 B, i64 H, i64 T, i64 d, i64 l, i64 c, double scale,
                      const float* q, const float* k, const float* v, i64 n, const i64* bh,
                      const i64* rows, double* o, double* lse, int nthreads) {
  Dims D{B, H, T, d};
  set_threads(nthreads);
#pragma omp parallel
  {
    std::vector<i64> s;
    std::vector<double> p;
#pragma omp for schedule(dynamic, 1)
    for (i64 r = 0; r < n; ++r) {
      i64 b = bh[r], i = rows[r], h = b % H;
      row_set(kind, mode, l, c, h, i, s);
      double L = row_softmax(rowp(q, D, b, i), k, D, b, scale, s, p);
      for (i64 x = 0; x < d; ++x) o[r * d + x] = 0.0;
      for (size_t t = 0; t < s.size(); ++t) {
        const float* vj = rowp(v, D, b, s[t]);
        for (i64 x = 0; x < d; ++x) o[r * d + x] += p[t] * (double)vj[x];
      }
      lse[r] = L;
    }
  }
}

// Backward over all heads. dq, dk, dv: [B,H,T,d] double, overwritten.
// For each row: P from the recomputed softmax, dP_ij = dO_i . v_j,
// D_i = sum_j P_ij dP_ij, dS_ij = P_ij (dP_ij - D_i);
// dq_i += scale dS_ij k_j, dk_j += scale dS_ij q_i, dv_j += P_ij dO_i.
void orc_backward(int kind, int mode, i64 B, i64 H, i64 T, i64 d, i64 l, i64 c, double scale,
                  const float* q, const float* k, const float* v, const float* dout, double* dq,
                  double* dk, double* dv, int nthreads) {
  Dims D{B, H, T, d};
  set_threads(nthreads);
  std::memset(dq, 0, sizeof(double) * B * H * T * d);
  std::memset(dk, 0, sizeof(double) * B * H * T * d);
  std::memset(dv, 0, sizeof(double) * B * H * T * d);
#pragma omp parallel
  {
    std::vector<i64> s;
    std::vector<double> p, dp;
#pragma omp for schedule(dynamic, 1)
    for (i64 b = 0; b < B * H; ++b) {
      i64 h = b % H;
      for (i64 i = 0; i < T; ++i) {
        row_set(kind, mode, l, c, h, i, s);
        if (s.empty()) continue;
        const float* qi = rowp(q, D, b, i);
        const float* doi = rowp(dout, D, b, i);
        row_softmax(qi, k, D, b, scale, s, p);
        dp.assign(s.size(), 0.0);
        double Di = 0.0;
        for (size_t t = 0; t < s.size(); ++t) {
          dp[t] = dot(doi, rowp(v, D, b, s[t]), d);
          Di += p[t] * dp[t];
        }
        double* dqi = dq + (b * T + i) * d;
        for (size_t t = 0; t < s.size(); ++t) {
          i64 j = s[t];
          double ds = p[t] * (dp[t] - Di);
          const float* kj = rowp(k, D, b, j);
          double* dkj = dk + (b * T + j) * d;
          double* dvj = dv + (b * T + j) * d;
          for (i64 x = 0; x < d; ++x) {
            dqi[x] += scale * ds * (double)kj[x];
            dkj[x] += scale * ds * (double)qi[x];
            dvj[x] += p[t] * (double)doi[x];
          }
        }
      }
    }
  }
}

// dQ for selected query rows (bh[r], rows[r]); dq: [n, d].
void orc_backward_query_rows(int kind, int mode, i64 B, i64 H, i64 T, i64 d, i64 l, i64 c,
                             double scale, const float* q, const float* k, const float* v,
                             const float* dout, i64 n, const i64* bh, const i64* rows, double* dq,
                             int nthreads) {
  Dims D{B, H, T, d};
  set_threads(nthreads);
#pragma omp parallel
  {
    std::vector<i64> s;
    std::vector<double> p, dp;
#pragma omp for schedule(dynamic, 1)
    for (i64 r = 0; r < n; ++r) {
      i64 b = bh[r], i = rows[r], h = b % H;
      for (i64 x = 0; x < d; ++x) dq[r * d + x] = 0.0;
      row_set(kind, mode, l, c, h, i, s);
      if (s.empty()) continue;
      const float* qi = rowp(q, D, b, i);
      const float* doi = rowp(dout, D, b, i);
      row_softmax(qi, k, D, b, scale, s, p);
      dp.assign(s.size(), 0.0);
      double Di = 0.0;
      for (size_t t = 0; t < s.size(); ++t) {
        dp[t] = dot(doi, rowp(v, D, b, s[t]), d);
        Di += p[t] * dp[t];
      }
      for (size_t t = 0; t < s.size(); ++t) {
        double ds = p[t] * (dp[t] - Di);
        const float* kj = rowp(k, D, b, s[t]);
        for (i64 x = 0; x < d; ++x) dq[r * d + x] += scale * ds * (double)kj[x];
      }
    }
  }
}

// dK, dV for selected key rows (bh[r], keys[r]): every query i >= j whose set
// holds j contributes; dk, dv: [n, d].
void orc_backward_key_rows(int kind, int mode, i64 B, i64 H, i64 T, i64 d, i64 l, i64 c,
                           double scale, const float* q, const float* k, const float* v,
                           const float* dout, i64 n, const i64* bh, const i64* keys, double* dk,
                           double* dv, int nthreads) {
  Dims D{B, H, T, d};
  set_threads(nthreads);
#pragma omp parallel
  {
    std::vector<i64> s;
    std::vector<double> p, dp;
#pragma omp for schedule(dynamic, 1)
    for (i64 r = 0; r < n; ++r) {
      i64 b = bh[r], j = keys[r], h = b % H;
      for (i64 x = 0; x < d; ++x) {
        dk[r * d + x] = 0.0;
        dv[r * d + x] = 0.0;
      }
      for (i64 i = j; i < T; ++i) {
        row_set(kind, mode, l, c, h, i, s);
        if (!row_has(s, j)) continue;
        const float* qi = rowp(q, D, b, i);
        const float* doi = rowp(dout, D, b, i);
        row_softmax(qi, k, D, b, scale, s, p);
        double Di = 0.0, pj = 0.0, dpj = 0.0;
        for (size_t t = 0; t < s.size(); ++t) {
          double dpt = dot(doi, rowp(v, D, b, s[t]), d);
          Di += p[t] * dpt;
          if (s[t] == j) {
            pj = p[t];
            dpj = dpt;
          }
        }
        double ds = pj * (dpj - Di);
        for (i64 x = 0; x < d; ++x) {
          dk[r * d + x] += scale * ds * (double)qi[x];
          dv[r * d + x] += pj * (double)doi[x];
        }
      }
    }
  }
}

}  // extern "C"

// ---- tile layout re-derived from the explicit sets ------------------------
//
// The CUDA library visits each head's set S_{h,i} in disjoint "segments",
// each with its own row order for queries and keys (a "view"):
//   view 0  natural order: position t;
//   view 1  summary gather (keys only): the last c positions of every
//           l-block, packed: sigma(j) = floor(j/l)*c + (j mod l) - (l-c);
//   view 2  residue-class order: t = p*l + r is row p of class r, view row
//           r*W + p. Classes of P = T/l rows are padded to W = a multiple of
//           128 rows, except short ones (8 <= P <= 64, P dividing 128), which
//           are packed (W = P: 128/P whole classes per tile).
// Tiles are 128 x 128 in view coordinates. This re-derivation walks every
// (i, j) pair of the explicit sets, assigns it to its segment and counts the
// pairs per tile; the library computes the same tiles from closed-form row
// intervals, and the tests require the two to agree bit for bit.
//
// Segment partition (the library's design, restated):
//   dense causal            : [nat/nat]
//   strided split, A1 head  : [nat/nat]
//   strided split, A2 head  : [cls/cls]                 (nat/nat if no class view)
//   strided merged          : [nat/nat: i-j <= l] + [cls/cls: i-j > l]
//   fixed split, A1 head    : [nat/nat]
//   fixed split, A2 head    : [nat/sum]                 (nat/nat if no summary view)
//   fixed merged            : [nat/nat: same block] + [nat/sum: earlier block]
// The class view exists when T mod l == 0 and l < T; the summary view also
// needs c | 128 and c <= l.

namespace {

const i64 TILE = 128;

struct ViewGeom {
  i64 T, l, c, P, ptiles, W;
};

bool has_cls(i64 T, i64 l) { return T % l == 0 && l < T; }
bool has_sum(i64 T, i64 l, i64 c) { return has_cls(T, l) && TILE % c == 0 && c <= l; }

int n_head_classes(int kind, int mode) { return (kind != DENSE_CAUSAL && mode == SPLIT) ? 2 : 1; }

int n_segments(int kind, int mode) {
  if (kind == DENSE_CAUSAL || mode == SPLIT) return 1;
  return 2;
}

// (qview, kview) of segment seg for head class hc.
void seg_views(int kind, int mode, i64 T, i64 l, i64 c, int hc, int seg, int* qv, int* kv) {
  *qv = 0;
  *kv = 0;
  if (kind == DENSE_CAUSAL) return;
  bool second = (mode == SPLIT) ? (hc == 1) : (seg == 1);
  if (!second) return;
  if (kind == STRIDED) {
    if (has_cls(T, l)) *qv = *kv = 2;
  } else {
    if (has_sum(T, l, c)) *kv = 1;
  }
}

// Segment of a live pair (i, j) of head class hc.
int seg_of(int kind, int mode, i64 l, i64 i, i64 j) {
  if (kind == DENSE_CAUSAL || mode == SPLIT) return 0;
  if (kind == STRIDED) return (i - j <= l) ? 0 : 1;
  return (j / l == i / l) ? 0 : 1;
}

i64 view_ntiles(int view, const ViewGeom& g) {
  if (view == 0) return (g.T + TILE - 1) / TILE;
  if (view == 1) return ((g.T / g.l) * g.c + TILE - 1) / TILE;
  return (g.l * g.W + TILE - 1) / TILE;
}

i64 view_tile(int view, const ViewGeom& g, i64 t) {
  if (view == 0) return t / TILE;
  if (view == 1) return ((t / g.l) * g.c + (t % g.l) - (g.l - g.c)) / TILE;
  return ((t % g.l) * g.W + t / g.l) / TILE;
}

}  // namespace

extern "C" {

int orc_num_head_classes(int kind, int mode) { return n_head_classes(kind, mode); }
int orc_num_segments(int kind, int mode) { return n_segments(kind, mode); }

void orc_segment_views(int kind, int mode, i64 T, i64 l, i64 c, int hc, int seg, int* qv, int* kv) {
  seg_views(kind, mode, T, l, c, hc, seg, qv, kv);
}

// Tiles of segment seg of head class hc (hc picks the even or odd heads in
// split mode), sorted by (query tile, key tile). Returns the tile count and
// writes at most cap triples. seg = -1 gives the plain natural-order tiling
// of the whole set (128 x 128 tiles of (i, j), no gather views).
i64 orc_layout_tiles(int kind, int mode, i64 T, i64 l, i64 c, int hc, int seg, i64* qt, i64* kt,
                     i64* live, i64 cap) {
  ViewGeom g{T, l, c, 0, 0, 0};
  if (has_cls(T, l)) {
    g.P = T / l;
    g.ptiles = (g.P + TILE - 1) / TILE;
    g.W = (g.P >= 8 && g.P <= 64 && TILE % g.P == 0) ? g.P : g.ptiles * TILE;
  }
  int qv = 0, kv = 0;
  if (seg >= 0) seg_views(kind, mode, T, l, c, hc, seg, &qv, &kv);
  i64 nq = view_ntiles(qv, g), nk = view_ntiles(kv, g);
  std::vector<i64> cnt((size_t)(nq * nk), 0);
  std::vector<i64> s;
  for (i64 i = 0; i < T; ++i) {
    row_set(kind, mode, l, c, hc, i, s);
    for (i64 j : s) {
      if (seg >= 0 && seg_of(kind, mode, l, i, j) != seg) continue;
      cnt[(size_t)(view_tile(qv, g, i) * nk + view_tile(kv, g, j))] += 1;
    }
  }
  i64 n = 0;
  for (i64 a = 0; a < nq; ++a) {
    for (i64 b = 0; b < nk; ++b) {
      i64 x = cnt[(size_t)(a * nk + b)];
      if (x == 0) continue;
      if (n < cap) {
        qt[n] = a;
        kt[n] = b;
        live[n] = x;
      }
      ++n;
    }
  }
  return n;
}

}  // extern "C"
