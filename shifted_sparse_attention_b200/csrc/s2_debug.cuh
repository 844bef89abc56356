// s2_debug.cuh -- bounds checks of the debug build of the library.
//
// Compiled with -DS2_DEBUG_BOUNDS (libs2attn_debug.so), every kernel checks,
// before it issues the access, each tile origin it computes against [0, N) and
// against the rows that may hold it (query tiles [q_begin, n_valid), key tiles
// [k_begin, n_valid)), each TMA row coordinate against the tensor, each global
// index it stores to, each stored-dS slot against the workspace, and the TMEM
// columns it addresses against the 512 allocated.  The first violation on the
// device is recorded in the status area (site, value, bounds) and the bounds
// flag is set; the access is skipped and the CTA aborts through the same
// bounded-wait path as a timeout.  Nothing traps.  In the normal build the
// checks compile to nothing.
#pragma once

namespace s2 {

// Status area (int[16] in device memory): [0] flag bits of the kernels;
// [1] a violation is recorded; [2] its site; long long [4..9] = value, lower
// bound (inclusive), upper bound (exclusive).
constexpr int kStatusInts = 16;
constexpr int kBoundsFlag = 0x1000;

// Check sites (s2attn_debug_bounds_report returns one of these).
enum BoundsSite {
  kSiteFwdQ = 1,      // forward: query tile origin / TMA row
  kSiteFwdKV = 2,     // forward: key (value) tile origin / TMA row
  kSiteFwdOut = 3,    // forward: O tile row, lse index
  kSiteFwdTmem = 4,   // forward: TMEM columns
  kSiteKvK = 5,       // dK/dV pass: key tile origin / TMA row
  kSiteKvQ = 6,       // dK/dV pass: query tile origin / TMA row, statistics rows
  kSiteKvDs = 7,      // dK/dV pass: stored-dS slot
  kSiteKvOut = 8,     // dK/dV pass: dK, dV tile row
  kSiteKvTmem = 9,    // dK/dV pass: TMEM columns
  kSiteDqQ = 10,      // dQ pass: query tile origin / TMA row, statistics index
  kSiteDqK = 11,      // dQ pass: key tile origin / TMA row, stored-dS slot
  kSiteDqOut = 12,    // dQ pass: dq tile row
  kSiteDqTmem = 13,   // dQ pass: TMEM columns
  kSiteProbe = 14,    // s2attn_debug_bounds_probe
};

#ifdef S2_DEBUG_BOUNDS
constexpr bool kBoundsChecked = true;
// Records the first violation and returns false.
static __device__ __noinline__ bool bounds_fail(int* status, int site, long long v, long long lo, long long hi) {
  atomicOr(status, kBoundsFlag);
  if (atomicCAS(status + 1, 0, 1) == 0) {
    status[2] = site;
    long long* r = reinterpret_cast<long long*>(status + 4);
    r[0] = v;
    r[1] = lo;
    r[2] = hi;
  }
  return false;
}
// True if lo <= v < hi; otherwise records the violation (needs `status` in scope).
#define S2_IN(site, v, lo, hi)                                                              \
  (((long long)(v) >= (long long)(lo) && (long long)(v) < (long long)(hi))                  \
       ? true                                                                                \
       : ::s2::bounds_fail(status, (site), (long long)(v), (long long)(lo), (long long)(hi)))
#else
constexpr bool kBoundsChecked = false;
#define S2_IN(site, v, lo, hi) true
#endif

}  // namespace s2
