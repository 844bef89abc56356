// Host replica of the kernels' traversal, built with g++ from the same
// scheduler header the CUDA kernels include (s2_index.cuh).  Used by
// tests/test_index_host.py to check the work decomposition and masks on the
// CPU against the oracle's visibility matrices, exhaustively for small N.
#include <cstdint>
#include <cstring>

#include "s2_index.cuh"

extern "C" {

// visited[i*N + j] += 1 for every (query i, key j) pair the kernels compute
// for a head of class `cls`; cover[i] += 1 for every query row a unit owns.
// Returns the number of work units decoded (non-idle).
int s2h_visit(int N, int G, int n_valid, int variant, int cls, uint8_t* visited, int32_t* cover) {
  s2::Plan p = s2::make_plan(1, N, 2, 128, G, n_valid, variant);
  int units = 0;
  for (int L = 0; L < s2::grid_fwd(p); ++L) {
    s2::Unit u;
    if (!s2::decode_unit(p, L, u)) continue;
    if (u.h != cls) continue;  // with H = 2, head h has class h (dense: head 0)
    ++units;
    for (int x = 0; x < 2; ++x) {
      if (u.t[x] < 0) continue;
      const int q0 = s2::tile_orig(p, u, u.t[x]);
      for (int r = 0; r < s2::kTile; ++r) cover[q0 + r] += 1;
      for (int k = 0; k <= u.kmax; ++k) {
        if (!s2::ktile_valid(p, u, k) || !s2::tile_takes(p, u, x, k)) continue;
        const int k0 = s2::tile_orig(p, u, k);
        for (int r = 0; r < s2::kTile; ++r) {
          const int lim = s2::col_limit(p, u, u.t[x], k, r);
          for (int c = 0; c < lim; ++c) visited[(size_t)(q0 + r) * N + (k0 + c)] += 1;
        }
      }
    }
  }
  return units;
}

// Same as s2h_visit for the backward's key-tile units: visited[i*N + j] += 1
// for every pair the backward computes; cover[j] += 1 per key row owned.
int s2h_visit_bwd(int N, int G, int n_valid, int variant, int cls, uint8_t* visited, int32_t* cover) {
  s2::Plan p = s2::make_plan(1, N, 2, 128, G, n_valid, variant);
  int units = 0;
  for (int L = 0; L < s2::grid_bwd(p); ++L) {
    s2::Unit u;
    if (!s2::decode_kv_unit(p, L, u)) continue;
    if (u.h != cls) continue;
    ++units;
    const int kt = u.t[0];
    const int k0 = s2::tile_orig(p, u, kt);
    for (int j = 0; j < s2::kTile; ++j) cover[k0 + j] += 1;
    if (!u.part[0]) continue;
    for (int qt = kt; qt <= u.kmax; ++qt) {
      if (!s2::ktile_valid(p, u, qt)) continue;
      const int q0 = s2::tile_orig(p, u, qt);
      for (int j = 0; j < s2::kTile; ++j) {
        int lo, hi;
        s2::query_range(p, u, kt, qt, j, lo, hi);
        for (int i = lo; i < hi; ++i) visited[(size_t)(q0 + i) * N + (k0 + j)] += 1;
      }
    }
  }
  return units;
}

// Traversals under a document mask (docs: per-position bounds [N][2], as the
// kernels read them), for the forward, the dK/dV pass and the dQ pass:
// visited[i*N + j] += 1 for every computed pair.  `which`: 0 forward, 1 dK/dV,
// 2 dQ.  docs == nullptr walks the plain graph.
int s2h_visit_docs(int N, int G, int n_valid, int variant, int cls, const int32_t* docs, int which,
                   uint8_t* visited) {
  s2::Plan p = s2::make_plan(1, N, 2, 128, G, n_valid, variant);
  p.docs = docs;
  int units = 0;
  if (which == 0) {
    for (int L = 0; L < s2::grid_fwd(p); ++L) {
      s2::Unit u;
      if (!s2::decode_unit(p, L, u) || u.h != cls) continue;
      ++units;
      for (int x = 0; x < 2; ++x) {
        if (!u.part[x]) continue;
        const int q0 = s2::tile_orig(p, u, u.t[x]);
        int lo, hi;
        s2::doc_span(p, u.b, q0, lo, hi);
        for (int k = 0; k <= u.t[x]; ++k) {
          if (!s2::ktile_valid(p, u, k) || !s2::tile_meets(s2::tile_orig(p, u, k), lo, hi)) continue;
          const int k0 = s2::tile_orig(p, u, k);
          for (int r = 0; r < s2::kTile; ++r) {
            int c0, c1;
            s2::row_cols(p, u, u.t[x], k, r, c0, c1);
            for (int c = c0; c < c1; ++c) visited[(size_t)(q0 + r) * N + (k0 + c)] += 1;
          }
        }
      }
    }
  } else if (which == 1) {
    for (int L = 0; L < s2::grid_bwd(p); ++L) {
      s2::Unit u;
      if (!s2::decode_kv_unit(p, L, u) || u.h != cls) continue;
      ++units;
      if (!u.part[0]) continue;
      const int kt = u.t[0], k0 = s2::tile_orig(p, u, kt);
      int lo, hi;
      s2::doc_span(p, u.b, k0, lo, hi);
      for (int qt = kt; qt <= u.kmax; ++qt) {
        if (!s2::ktile_valid(p, u, qt) || !s2::tile_meets(s2::tile_orig(p, u, qt), lo, hi)) continue;
        const int q0 = s2::tile_orig(p, u, qt);
        for (int j = 0; j < s2::kTile; ++j) {
          int a, b;
          s2::key_cols(p, u, kt, qt, j, a, b);
          for (int i = a; i < b; ++i) visited[(size_t)(q0 + i) * N + (k0 + j)] += 1;
        }
      }
    }
  } else {
    for (int L = 0; L < s2::grid_bwd(p); ++L) {
      s2::Unit u;
      if (!s2::decode_q_unit(p, L, u) || u.h != cls) continue;
      ++units;
      if (!u.part[0]) continue;
      const int qt = u.t[0], q0 = s2::tile_orig(p, u, qt);
      int lo, hi;
      s2::doc_span(p, u.b, q0, lo, hi);
      for (int k = 0; k <= qt; ++k) {
        if (!s2::ktile_valid(p, u, k) || !s2::tile_meets(s2::tile_orig(p, u, k), lo, hi)) continue;
        const int k0 = s2::tile_orig(p, u, k);
        for (int r = 0; r < s2::kTile; ++r) {
          int c0, c1;
          s2::row_cols(p, u, qt, k, r, c0, c1);
          for (int c = c0; c < c1; ++c) visited[(size_t)(q0 + r) * N + (k0 + c)] += 1;
        }
      }
    }
  }
  return units;
}

// Sequence-parallel traversal: the pairs computed by rank `rank` of `world`
// (shards of L rows, plan over the extended buffer of s + L rows whose first
// s rows are the halo), mapped to GLOBAL positions of the N = world·L
// sequence: extended row e is global rank·L - s + e (modulo N for ROLLED).
// visited[gi*N + gj] += 1 per computed pair; `which`: 0 forward, 1 dK/dV,
// 2 dQ (each walk mirrors its kernel's traversal).  Returns -1 if a pair
// touches a halo row with no global position (rank 0 of STRICT).
int s2h_visit_sp(int L, int G, int n_valid_local, int variant, int rank, int world, int cls, int which,
                 uint8_t* visited) {
  const int s = G / 2, N = world * L;
  s2::Plan p = s2::make_plan_sp(1, L, 2, 128, G, s + n_valid_local, variant == s2::kStrict && rank == 0);
  int bad = 0;
  auto mark = [&](int qe, int ke) {
    long long gq = (long long)rank * L - s + qe, gk = (long long)rank * L - s + ke;
    if (variant == s2::kRolled) { gq = (gq + N) % N; gk = (gk + N) % N; }
    if (gq < 0 || gk < 0 || gq >= N || gk >= N) { bad = 1; return; }
    visited[gq * N + gk] += 1;
  };
  if (which == 0) {
    for (int Li = 0; Li < s2::grid_fwd(p); ++Li) {
      s2::Unit u;
      if (!s2::decode_unit(p, Li, u) || u.h != cls) continue;
      for (int x = 0; x < 2; ++x) {
        if (!u.part[x]) continue;
        const int q0 = s2::tile_orig(p, u, u.t[x]);
        for (int k = 0; k <= u.t[x]; ++k) {
          if (!s2::ktile_valid(p, u, k)) continue;
          const int k0 = s2::tile_orig(p, u, k);
          for (int r = 0; r < s2::kTile; ++r) {
            const int lim = s2::col_limit(p, u, u.t[x], k, r);
            for (int c = 0; c < lim; ++c) mark(q0 + r, k0 + c);
          }
        }
      }
    }
  } else if (which == 1) {
    for (int Li = 0; Li < s2::grid_bwd(p); ++Li) {
      s2::Unit u;
      if (!s2::decode_kv_unit(p, Li, u) || u.h != cls || !u.part[0]) continue;
      const int kt = u.t[0], k0 = s2::tile_orig(p, u, kt);
      for (int qt = kt; qt <= u.kmax; ++qt) {  // the kernel starts at the first valid query tile
        if (!s2::qtile_valid(p, u, qt)) continue;
        const int q0 = s2::tile_orig(p, u, qt);
        for (int j = 0; j < s2::kTile; ++j) {
          int lo, hi;
          s2::query_range(p, u, kt, qt, j, lo, hi);
          for (int i = lo; i < hi; ++i) mark(q0 + i, k0 + j);
        }
      }
    }
  } else {
    for (int Li = 0; Li < s2::grid_bwd(p); ++Li) {
      s2::Unit u;
      if (!s2::decode_q_unit(p, Li, u) || u.h != cls || !u.part[0]) continue;
      const int qt = u.t[0], q0 = s2::tile_orig(p, u, qt);
      for (int k = 0; k <= qt; ++k) {
        if (!s2::ktile_valid(p, u, k)) continue;
        const int k0 = s2::tile_orig(p, u, k);
        for (int r = 0; r < s2::kTile; ++r) {
          const int lim = s2::col_limit(p, u, qt, k, r);
          for (int c = 0; c < lim; ++c) mark(q0 + r, k0 + c);
        }
      }
    }
  }
  return bad ? -1 : 0;
}

// Stored-dS tile slots: writes[slot] += 1 for every tile pair the dK/dV pass
// computes (key tile units, query tiles from the first valid one, under the
// document spans), reads[slot] += 1 for every tile pair the dQ pass reads.
// Returns B·H·ds_head_tiles (the slot count of the workspace) or -1 if a slot
// falls outside it.
long long s2h_ds_slots(int B, int N, int H, int G, int n_valid, int variant, const int32_t* docs, int32_t* writes,
                       int32_t* reads) {
  s2::Plan p = s2::make_plan(B, N, H, 128, G, n_valid, variant);
  p.docs = docs;
  const long long total = (long long)B * H * p.ds_head_tiles;
  bool bad = false;
  for (int Li = 0; Li < s2::grid_bwd(p); ++Li) {
    s2::Unit u;
    if (!s2::decode_kv_unit(p, Li, u) || !u.part[0]) continue;
    const int kt = u.t[0];
    int lo, hi;
    s2::doc_span(p, u.b, s2::tile_orig(p, u, kt), lo, hi);
    for (int qt = kt; qt <= u.kmax; ++qt) {
      if (!s2::qtile_valid(p, u, qt) || !s2::tile_meets(s2::tile_orig(p, u, qt), lo, hi)) continue;
      const long long sl = s2::ds_slot(p, u, qt, kt);
      if (sl < 0 || sl >= total) bad = true; else writes[sl] += 1;
    }
  }
  for (int Li = 0; Li < s2::grid_bwd(p); ++Li) {
    s2::Unit u;
    if (!s2::decode_q_unit(p, Li, u) || !u.part[0]) continue;
    const int qt = u.t[0];
    int lo, hi;
    s2::doc_span(p, u.b, s2::tile_orig(p, u, qt), lo, hi);
    for (int k = 0; k <= qt; ++k) {
      if (!s2::ktile_valid(p, u, k) || !s2::tile_meets(s2::tile_orig(p, u, k), lo, hi)) continue;
      const long long sl = s2::ds_slot(p, u, qt, k);
      if (sl < 0 || sl >= total) bad = true; else reads[sl] += 1;
    }
  }
  return bad ? -1 : total;
}

// Grid size and per-class unit counts of a launch.
void s2h_plan(int B, int N, int H, int G, int n_valid, int variant, int32_t* out) {
  s2::Plan p = s2::make_plan(B, N, H, 128, G, n_valid, variant);
  out[0] = s2::grid_fwd(p);
  out[1] = p.nseg[0];
  out[2] = p.nseg[1];
  out[3] = p.nunit[0];
  out[4] = p.nunit[1];
}
}
