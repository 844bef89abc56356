// s2_index.cuh -- S²-Attn segment / tile scheduler and mask predicates,
// shared by the host launcher and every kernel (forward, backward, adjacency
// dump), so that all of them visit exactly the same (query, key) pairs.
//
// Method ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调", §1 "S²-Attn的计算图"):
//   heads [0, H/2) group positions by b(i) = floor(i/G); heads [H/2, H) shift
//   by s = G/2 and group by b'(i) = floor((i - s)/G); attention is causal
//   inside a group; the shifted heads' outputs go back to original positions.
//   Boundary variants of the shifted heads (same section):
//     STRICT  -- separate short head group [0, s) and tail group [N - s, N);
//     ROLLED  -- roll left by s and keep the in-group triangular mask, so the
//                last group is [N - s, N) followed by [0, s);
//   DENSE_CAUSAL is the full causal graph used at inference (§2).
//   The reshape [B, N, H, D] -> [B*M, G, H, D] of §1 becomes index math here:
//   no tensor is ever rolled or copied.
//
// Virtual coordinates.  For every (head class, variant) the rows of a head
// are laid out in a "virtual" order in which each segment is a contiguous
// range and causality is "virtual key <= virtual query":
//   class 0, STRICT class 1, DENSE: virtual index = original position;
//   ROLLED class 1: virtual index r = rolled position, original = (r + s) mod N.
// With s a multiple of 128, every 128-row tile of virtual rows is a
// contiguous range of original positions, so each tile is one TMA box.
//
// Segment lattice.  Outside DENSE_CAUSAL, the segments of class c are the
// intervals [off_c + kG, off_c + (k+1)G) of virtual rows clipped to [0, N):
// off = {0, s} gives STRICT (the clipped first and last intervals are its
// short head and tail groups), off = {0, 0} gives class 0 and the rolled
// coordinates of ROLLED class 1.
//
// Sequence parallelism ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1,
// distributed boundaries: the shifted heads exchange a half-group halo with
// the neighbouring rank): a rank holding the G-aligned shard [rL, rL + L) of a
// STRICT (or ROLLED) sequence works on an extended buffer of N = s + L rows
// whose first s rows are the halo, rows [rL - s, rL) of the previous rank.
// In those coordinates class 0's boundaries sit at s + kG and class 1's at
// kG, i.e. off = {s, 0}; halo rows are keys only (q_begin = s), and on the
// first rank of a STRICT sequence they hold no key at all (k_begin = s).
#pragma once
#include <cstdint>

#ifdef __CUDACC__
#define S2_HD __host__ __device__ __forceinline__
#else
#define S2_HD inline
#endif

namespace s2 {

constexpr int kTile = 128;  // rows per query tile and per key tile

enum Variant { kStrict = 0, kRolled = 1, kDenseCausal = 2 };

struct Plan {
  int B, N, H, D, G, s, n_valid, variant;
  int nseg[2];     // segments per head class
  int nunit[2];    // max work units (pairs of q tiles) per segment, per class
  int ranks;       // max over classes of nseg * nunit (forward grid = ranks * B * H)
  int ntile[2];    // max tiles per segment, per class
  int kv_ranks;    // max over classes of nseg * ntile (grid of each backward pass = kv_ranks * B * H)
  int hg_fwd, hg_bwd;  // heads interleaved per group of consecutive CTAs (L2 locality)
  int off[2];      // segment lattice offset per class (see above)
  int q_begin;     // rows [0, q_begin) are never queries (a sequence-parallel halo)
  int k_begin;     // rows [0, k_begin) hold no valid key
  long long ds_head_tiles;  // 128x128 dS tiles per (b, h) in the stored-dS backward
  int nquad[2];    // CTA-pair forward: units of four query tiles per segment, per class
  int quad_ranks;  // max over classes of nseg * nquad (CTA-pair forward: clusters per head)
  float scale_log2;  // log2(e) / sqrt(D)
  // Packed sequences: per-position document bounds [B, N, 2] = {first position,
  // one past the last position} of the position's document (original
  // positions), or null when the sequence is one document.
  const int* docs;
};

// Linear CTA index -> (flattened head bh, per-head slot r).  CTAs are issued
// in groups of `hg` heads; inside a group the slot r is the slow index, so the
// CTAs resident at one time work on few heads and their K/V (forward) or
// Q/dO and dq rows (backward) stay in L2, while r still runs longest-first.
S2_HD bool split_index(const Plan& p, int L, int R, int hg, int& bh, int& r) {
  const int BH = p.B * p.H;
  const int grp = L / (hg * R), within = L % (hg * R);
  r = within / hg;
  bh = grp * hg + within % hg;
  return bh < BH;
}

S2_HD int groups_of(int n, int hg) { return (n + hg - 1) / hg; }

S2_HD int head_class(const Plan& p, int h) {
  return (p.variant == kDenseCausal) ? 0 : (h >= p.H / 2 ? 1 : 0);
}

S2_HD int seg_count(const Plan& p, int cls) {
  if (p.variant == kDenseCausal) return 1;
  const int o = p.off[cls];
  return (o ? 1 : 0) + (p.N - o + p.G - 1) / p.G;
}

// Virtual range [vbeg, vbeg + len) of segment `seg`.
S2_HD void seg_bounds(const Plan& p, int cls, int seg, int& vbeg, int& len) {
  if (p.variant == kDenseCausal) { vbeg = 0; len = p.N; return; }
  const int o = p.off[cls];
  if (o && seg == 0) { vbeg = 0; len = o; return; }
  vbeg = o + (seg - (o ? 1 : 0)) * p.G;
  len = p.N - vbeg < p.G ? p.N - vbeg : p.G;
}

// Segment containing virtual row v.
S2_HD int seg_of(const Plan& p, int cls, int v) {
  if (p.variant == kDenseCausal) return 0;
  const int o = p.off[cls];
  if (v < o) return 0;
  return (v - o) / p.G + (o ? 1 : 0);
}

S2_HD int orig_of(const Plan& p, int cls, int v) {
  if (cls == 1 && p.variant == kRolled) {
    int o = v + p.s;
    return o >= p.N ? o - p.N : o;
  }
  return v;
}

S2_HD int virt_of(const Plan& p, int cls, int x) {
  if (cls == 1 && p.variant == kRolled) {
    int v = x - p.s;
    return v < 0 ? v + p.N : v;
  }
  return x;
}

// One CTA work unit: up to two consecutive query tiles of one segment.
struct Unit {
  int b, h, cls;
  int seg;         // segment index within the head class
  int vbeg;        // virtual start of the segment
  int ntiles;      // query tiles in the segment
  int t[2];        // local tile indices (t[1] = -1 if absent)
  bool part[2];    // tile exists and holds at least one valid row
  int kmax;        // largest key tile index any participating tile needs (-1: none)
};

// Original position of the first row of local tile `t` of the unit's segment.
S2_HD int tile_orig(const Plan& p, const Unit& u, int t) {
  return orig_of(p, u.cls, u.vbeg + t * kTile);
}

// A key tile is processed iff it holds at least one valid key; a query tile
// iff it holds at least one valid query row.  (n_valid cuts inside a tile;
// q_begin and k_begin are multiples of the tile.)
S2_HD bool ktile_valid(const Plan& p, const Unit& u, int k) {
  const int x0 = tile_orig(p, u, k);
  return x0 >= p.k_begin && x0 < p.n_valid;
}
S2_HD bool qtile_valid(const Plan& p, const Unit& u, int t) {
  const int x0 = tile_orig(p, u, t);
  return x0 >= p.q_begin && x0 < p.n_valid;
}

// Decode a linear work index (longest work first).  Returns false for idle indices.
S2_HD bool decode_unit(const Plan& p, int L, Unit& u) {
  int bh, r;
  if (!split_index(p, L, p.ranks, p.hg_fwd, bh, r)) return false;
  u.b = bh / p.H;
  u.h = bh % p.H;
  u.cls = head_class(p, u.h);
  const int S = p.nseg[u.cls], NU = p.nunit[u.cls];
  if (r >= S * NU) return false;
  const int unit = NU - 1 - r / S;
  const int seg = r % S;
  u.seg = seg;
  int len;
  seg_bounds(p, u.cls, seg, u.vbeg, len);
  u.ntiles = len / kTile;
  if (2 * unit >= u.ntiles) return false;
  u.t[0] = 2 * unit;
  u.t[1] = (2 * unit + 1 < u.ntiles) ? 2 * unit + 1 : -1;
  u.kmax = -1;
  for (int x = 0; x < 2; ++x) {
    u.part[x] = (u.t[x] >= 0) && qtile_valid(p, u, u.t[x]);
    if (u.part[x]) u.kmax = u.t[x];
  }
  return true;
}

// Query tile x takes part at key tile k.
S2_HD bool tile_takes(const Plan& p, const Unit& u, int x, int k) {
  return u.part[x] && k <= u.t[x];
}

// Number of key columns of key tile k visible from local row r (0..127) of
// query tile tq: columns [0, limit) are visible, the rest masked.  Combines
// the causal triangle of the diagonal tile with the padding mask on keys and
// on the query row (positions >= n_valid).
S2_HD int col_limit(const Plan& p, const Unit& u, int tq, int k, int r) {
  const int q0 = tile_orig(p, u, tq);
  if (q0 + r >= p.n_valid) return 0;
  int lim = (k == tq) ? r + 1 : kTile;
  const int kv = p.n_valid - tile_orig(p, u, k);
  return lim < kv ? lim : kv;
}

// ---------------------------------------------------------------- backward units
// The backward runs one CTA per key tile (128 keys) of a segment and walks the
// query tiles from the diagonal to the end of the segment.  The unit reuses
// Unit: t[0] = key tile, t[1] = -1, part[0] = the key tile holds a valid key,
// kmax = last query tile of the segment.

// Decode a linear backward work index (key tiles with the most query tiles first).
S2_HD bool decode_kv_unit(const Plan& p, int L, Unit& u) {
  int bh, r;
  if (!split_index(p, L, p.kv_ranks, p.hg_bwd, bh, r)) return false;
  u.b = bh / p.H;
  u.h = bh % p.H;
  u.cls = head_class(p, u.h);
  const int S = p.nseg[u.cls], NT = p.ntile[u.cls];
  if (r >= S * NT) return false;
  const int kt = r / S, seg = r % S;
  u.seg = seg;
  int len;
  seg_bounds(p, u.cls, seg, u.vbeg, len);
  u.ntiles = len / kTile;
  if (kt >= u.ntiles) return false;
  u.t[0] = kt;
  u.t[1] = -1;
  u.part[0] = ktile_valid(p, u, kt);
  u.part[1] = false;
  u.kmax = u.ntiles - 1;
  return true;
}

// Decode a linear dq-pass work index: one query tile of a segment, whose key
// tiles run from the segment start to the diagonal (query tiles with the
// most key tiles first).  Unit: t[0] = query tile, part[0] = it holds a valid
// row, kmax = t[0].
S2_HD bool decode_q_unit(const Plan& p, int L, Unit& u) {
  int bh, r;
  if (!split_index(p, L, p.kv_ranks, p.hg_bwd, bh, r)) return false;
  u.b = bh / p.H;
  u.h = bh % p.H;
  u.cls = head_class(p, u.h);
  const int S = p.nseg[u.cls], NT = p.ntile[u.cls];
  if (r >= S * NT) return false;
  const int rank = r / S, seg = r % S;
  u.seg = seg;
  int len;
  seg_bounds(p, u.cls, seg, u.vbeg, len);
  u.ntiles = len / kTile;
  const int qt = u.ntiles - 1 - rank;
  if (qt < 0) return false;
  u.t[0] = qt;
  u.t[1] = -1;
  u.part[0] = qtile_valid(p, u, qt);
  u.part[1] = false;
  u.kmax = qt;
  return true;
}

// Queries of query tile qt visible from local key row j of key tile kt:
// columns [lo, hi).  The same set as col_limit, seen from the key side.
S2_HD void query_range(const Plan& p, const Unit& u, int kt, int qt, int j, int& lo, int& hi) {
  lo = (kt == qt) ? j : 0;
  if (tile_orig(p, u, kt) + j >= p.n_valid) { hi = 0; return; }
  const int qv = p.n_valid - tile_orig(p, u, qt);
  hi = qv < kTile ? qv : kTile;
}

// ---------------------------------------------------------------- stored dS
// The stored-dS backward keeps every computed 128x128 tile of dS (bf16) from
// the dK/dV pass for the dQ pass.  Tile (query tile qt, key tile kt <= qt) of
// a segment sits at slot tri(qt) + kt of the segment's triangle; segments of
// a head follow each other, heads follow each other (ds_head_tiles apart).
// A tile is stored transposed, row = key, column = query, as the dK/dV pass
// produces it (thread = key row).
S2_HD long long tri(int n) { return (long long)n * (n + 1) / 2; }

S2_HD long long ds_seg_base(const Plan& p, int cls, int seg) {
  if (p.variant == kDenseCausal) return 0;
  const int o = p.off[cls], T = p.G / kTile;
  if (!o) return (long long)seg * tri(T);
  return seg == 0 ? 0 : tri(o / kTile) + (long long)(seg - 1) * tri(T);
}

S2_HD long long ds_slot(const Plan& p, const Unit& u, int qt, int kt) {
  return ((long long)u.b * p.H + u.h) * p.ds_head_tiles + ds_seg_base(p, u.cls, u.seg) + tri(qt) + kt;
}

// Grid sizes of the forward and backward launches.
S2_HD int grid_fwd(const Plan& p) { return groups_of(p.B * p.H, p.hg_fwd) * p.hg_fwd * p.ranks; }
S2_HD int grid_bwd(const Plan& p) { return groups_of(p.B * p.H, p.hg_bwd) * p.hg_bwd * p.kv_ranks; }

// ---------------------------------------------------------------- document mask
// Packed sequences ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1): key j
// is visible from query i only if both lie in the same document, for both head
// classes.  Documents are contiguous runs of original positions, so the keys
// of i's document form the range [doc_lo(i), doc_hi(i)), and a query tile and
// a key tile (each a contiguous range of original positions) hold a pair in
// the same document iff the key tile meets the span of the documents that
// touch the query tile (and symmetrically).

S2_HD int doc_lo(const Plan& p, int b, int x) { return p.docs[(((long long)b * p.N) + x) * 2]; }
S2_HD int doc_hi(const Plan& p, int b, int x) { return p.docs[(((long long)b * p.N) + x) * 2 + 1]; }

// Span [lo, hi) of the documents touching the tile of 128 rows starting at
// original position x0 (everything when there are no documents).
S2_HD void doc_span(const Plan& p, int b, int x0, int& lo, int& hi) {
  if (!p.docs) { lo = 0; hi = p.N; return; }
  lo = doc_lo(p, b, x0);
  hi = doc_hi(p, b, x0 + kTile - 1);
}

// The tile of 128 positions starting at x0 meets the span [lo, hi).
S2_HD bool tile_meets(int x0, int lo, int hi) { return x0 < hi && x0 + kTile > lo; }

// Key columns [cmin, cmax) of key tile k visible from row r of query tile tq:
// the causal diagonal, padding, and the row's document.
S2_HD void row_cols(const Plan& p, const Unit& u, int tq, int k, int r, int& cmin, int& cmax) {
  cmin = 0;
  cmax = col_limit(p, u, tq, k, r);
  if (p.docs && cmax > 0) {
    const int k0 = tile_orig(p, u, k), x = tile_orig(p, u, tq) + r;
    const int lo = doc_lo(p, u.b, x) - k0, hi = doc_hi(p, u.b, x) - k0;
    if (lo > cmin) cmin = lo;
    if (hi < cmax) cmax = hi;
  }
}

// Query columns [lo, hi) of query tile qt visible from key row j of key tile
// kt (the same set as row_cols, seen from the key side).
S2_HD void key_cols(const Plan& p, const Unit& u, int kt, int qt, int j, int& lo, int& hi) {
  query_range(p, u, kt, qt, j, lo, hi);
  if (p.docs && hi > lo) {
    const int q0 = tile_orig(p, u, qt), y = tile_orig(p, u, kt) + j;
    const int dl = doc_lo(p, u.b, y) - q0, dh = doc_hi(p, u.b, y) - q0;
    if (dl > lo) lo = dl;
    if (dh < hi) hi = dh;
  }
}

// Per-class unit and tile counts of a plan whose geometry is set.
inline void finish_plan(Plan& p) {
  for (int c = 0; c < 2; ++c) {
    p.nseg[c] = seg_count(p, c);
    int maxlen = 0;
    for (int sgi = 0; sgi < p.nseg[c]; ++sgi) {
      int vb, len;
      seg_bounds(p, c, sgi, vb, len);
      if (len > maxlen) maxlen = len;
    }
    const int nt = maxlen / kTile;
    p.nunit[c] = (nt + 1) / 2;
    p.ntile[c] = nt;
  }
  for (int c = 0; c < 2; ++c) p.nquad[c] = (p.ntile[c] + 3) / 4;
  const int q0 = p.nseg[0] * p.nquad[0], q1 = p.nseg[1] * p.nquad[1];
  p.quad_ranks = q0 > q1 ? q0 : q1;
  const int r0 = p.nseg[0] * p.nunit[0], r1 = p.nseg[1] * p.nunit[1];
  p.ranks = r0 > r1 ? r0 : r1;
  const int k0 = p.nseg[0] * p.ntile[0], k1 = p.nseg[1] * p.ntile[1];
  p.kv_ranks = k0 > k1 ? k0 : k1;
  p.hg_fwd = 2;
  p.hg_bwd = 1;
  p.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)p.D));
  // stored-dS tiles per head: the larger class's sum over segments of tri(tiles)
  p.ds_head_tiles = 0;
  for (int c = 0; c < 2; ++c) {
    long long t = 0;
    for (int sgi = 0; sgi < p.nseg[c]; ++sgi) {
      int vb, len;
      seg_bounds(p, c, sgi, vb, len);
      t += tri(len / kTile);
    }
    if (t > p.ds_head_tiles) p.ds_head_tiles = t;
  }
}

// Host-side plan construction (validated by the caller).
inline Plan make_plan(int B, int N, int H, int D, int G, int n_valid, int variant) {
  Plan p{};
  p.B = B; p.N = N; p.H = H; p.D = D; p.G = G; p.s = G / 2;
  p.n_valid = n_valid; p.variant = variant;
  p.off[0] = 0;
  p.off[1] = (variant == kStrict) ? p.s : 0;
  p.q_begin = 0;
  p.k_begin = 0;
  p.docs = nullptr;
  finish_plan(p);
  return p;
}

// Plan of one sequence-parallel rank over its extended buffer of s + L rows
// (halo first).  n_valid counts extended rows; first_strict: the rank holds
// the start of a STRICT sequence, so its halo rows are not keys.
inline Plan make_plan_sp(int B, int L, int H, int D, int G, int n_valid, bool first_strict) {
  Plan p{};
  p.B = B; p.H = H; p.D = D; p.G = G; p.s = G / 2;
  p.N = p.s + L;
  p.n_valid = n_valid;
  p.variant = kStrict;  // plain (unrolled) coordinates in the extended buffer
  p.off[0] = p.s;
  p.off[1] = 0;
  p.q_begin = p.s;
  p.k_begin = first_strict ? p.s : 0;
  p.docs = nullptr;
  finish_plan(p);
  return p;
}

}  // namespace s2
