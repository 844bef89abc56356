// s2_fwd2.cu -- S²-Attn forward over CTA pairs (tcgen05 cta_group::2), D = 128.
//
// Same result as s2_fwd.cu ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调", §3:
// softmax attention over each row's visible set S_i of §1), with the products
// issued for a pair of CTAs at once (M = 256 rows): each score MMA
// S = Q K^T reads its own 128 query rows and HALF of the key tile from each
// CTA's shared memory, and O += P V reads P from each CTA's tensor memory and
// half of the value columns from each CTA.  Per product a CTA's shared memory
// delivers 6 KB instead of 8 KB, per key tile a CTA loads 32 KB of K/V
// instead of 64 KB, and one thread issues the MMAs for both CTAs: the score
// MMAs of the single-CTA kernel, with both operands in shared memory, run at
// the SM's shared-memory bandwidth, which this layout relieves.  Measured on the
// long-context workload it is nevertheless slower (2.97 against 2.25 ms): a
// pair product still takes 72-79 cycles to issue, and each tile's hand-off now
// waits for the slower softmax of two CTAs.  It is an option, off by default.
//
// A cluster of two CTAs owns four consecutive 128-row query tiles of one
// segment: CTA r holds tiles A = 4w + r and B = 4w + 2 + r, so the "A pair"
// (4w, 4w+1) and the "B pair" (4w+2, 4w+3) each form one M = 256 product.
// A pair works through the key tiles up to its later tile's diagonal; for
// the earlier tile's CTA the last one is masked out entirely (P = 0).
// Roles per CTA (320 threads): warps 0-3 / 4-7 softmax of tiles A / B (thread
// = row = TMEM lane), warp 8 TMA producer (own Q tiles; own halves of every
// K and V tile), warp 9 TMEM allocator; in CTA 0 one thread of warp 9 issues
// all MMAs.  Handshakes:
//   K/V, Q loads of both CTAs complete on CTA 0's barriers (.cta_group::2
//     TMA; CTA 0's producer announces the bytes of both halves);
//   P_FULL(x): each of the pair's 8 warps of softmax warpgroup x arrives once on
//     CTA 0's barrier;
//   S_FULL, KV_EMPTY, MMA_DONE: tcgen05.commit to the barrier of each CTA;
//   EXIT: each CTA tells the other it has read its accumulators, before the
//     paired TMEM allocation is released.
// Every wait is bounded (s2_wait / s2_wait_cl).  No TMA load uses multicast.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_index.cuh"
#include "s2_kernels.h"
#include "sm100_ptx.cuh"

namespace s2 {

namespace fwd2 {

constexpr int D = 128;
constexpr int kThreads = 320;
constexpr int kSlots = 10;                          // 16 KB halves of K or V tiles
constexpr int kQBytes = kTile * D * 2;              // 32 KB
constexpr int kHalfBytes = kTile * D;               // 16 KB: half a K or V tile
constexpr int kQChunk = kTile * 64 * 2;             // 128 rows x 64 columns
constexpr int kKChunk = 64 * 64 * 2;                // 64 rows x 64 columns (half a K tile's chunk)

enum Bar {
  KV_FULL = 0,     // + slot (10), used in CTA 0
  KV_EMPTY = 10,   // + slot (10)
  S_FULL = 20,     // + tile (2)
  P_FULL = 22,     // + tile (2), used in CTA 0
  Q_FULL = 24,     // used in CTA 0
  MMA_DONE = 25,
  EXIT = 26,
  NUM_BARS = 27
};

struct Layout {
  static constexpr int kQ = 0;
  static constexpr int kKV = 2 * kQBytes;
  static constexpr int kBars = kKV + kSlots * kHalfBytes;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

// ---------------------------------------------------------------- cluster PTX
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cl_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cl_addr), "r"(v) : "memory");
}
// Bounded wait with cluster-scope acquire (arrivals may come from the peer CTA).
// A timeout sets the abort flag of both CTAs (peer_abort: the peer's flag, as a
// shared::cluster address), so that every role of the pair gives up promptly and
// both reach the exit handshake.
__device__ __forceinline__ bool s2_wait_cl(uint32_t bar, uint32_t parity, volatile int* abort, int* status,
                                           int code, uint32_t peer_abort) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitBudgetCycles) {
      *abort = 1;
      st_cluster_u32(peer_abort, 1u);
      atomicOr(status, code);
      return false;
    }
  }
}
// The exit handshake's wait ignores the abort flag: a CTA must not retire while
// its peer may still reach its shared memory.  Its budget covers the peer's
// longest way there (one timed-out wait, the others cut short by the flag).
__device__ __forceinline__ void wait_exit(uint32_t bar, int* status) {
  const long long t0 = clock64();
  while (!mbar_try_wait_cl(bar, 0)) {
    if (clock64() - t0 > 4 * kWaitBudgetCycles) {
      atomicOr(status, 64);
      return;
    }
  }
}
// 3-D tiled load into this CTA's shared memory whose bytes complete on a barrier
// of either CTA of the pair (cl_bar: shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void* tmap, int c0, int c1, int c2,
                                                 uint32_t cl_bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(cl_bar)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrive on barrier `bar` (same offset) of both CTAs once the issued MMAs
// complete: one commit per CTA, the peer's barrier named by its cluster address.
__device__ __forceinline__ void umma_commit_to(uint32_t cl_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(cl_bar)
               : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  umma_commit_to(map_to(bar, 0));
  umma_commit_to(map_to(bar, 1));
}

// A cluster's work: four consecutive query tiles of one segment.
struct Quad {
  Unit u;          // b, h, cls, seg, vbeg, ntiles; t[x] = this CTA's tiles (may lie past the segment)
  bool own[2];     // this CTA's tile x exists and holds a valid row
  bool pair[2];    // pair x (this CTA's tile x and the peer's) has a valid row
  int kmax[2];     // last key tile of pair x (its later valid tile's diagonal)
};

__device__ __forceinline__ bool decode_quad(const Plan& p, int cluster, int rank, Quad& q) {
  int bh, r;
  if (!split_index(p, cluster, p.quad_ranks, p.hg_fwd, bh, r)) return false;
  Unit& u = q.u;
  u.b = bh / p.H;
  u.h = bh % p.H;
  u.cls = head_class(p, u.h);
  const int S = p.nseg[u.cls], NQ = p.nquad[u.cls];
  if (r >= S * NQ) return false;
  const int w = NQ - 1 - r / S;
  u.seg = r % S;
  int len;
  seg_bounds(p, u.cls, u.seg, u.vbeg, len);
  u.ntiles = len / kTile;
  if (4 * w >= u.ntiles) return false;
  for (int x = 0; x < 2; ++x) {
    q.kmax[x] = -1;
    for (int c = 0; c < 2; ++c) {  // the pair's two tiles, in order
      const int t = 4 * w + 2 * x + c;
      const bool v = t < u.ntiles && qtile_valid(p, u, t);
      if (c == rank) q.own[x] = v;
      if (v) q.kmax[x] = t;
    }
    q.pair[x] = q.kmax[x] >= 0;
    u.t[x] = 4 * w + 2 * x + rank;
    u.part[x] = q.own[x];
  }
  u.kmax = q.kmax[1] > q.kmax[0] ? q.kmax[1] : q.kmax[0];
  return true;
}

__device__ __forceinline__ bool pair_takes(const Quad& q, int x, int k) { return q.pair[x] && k <= q.kmax[x]; }

__device__ __forceinline__ int next_key(const Plan& p, const Quad& q, int k) {
  for (int j = k + 1; j <= q.u.kmax; ++j)
    if (ktile_valid(p, q.u, j) && (pair_takes(q, 0, j) || pair_takes(q, 1, j))) return j;
  return -1;
}

}  // namespace fwd2

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(fwd2::kThreads, 1)
    s2_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK64,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ Plan p, float* __restrict__ lse, int* __restrict__ status) {
  using namespace fwd2;
  using L = fwd2::Layout;
  const uint32_t rank = cluster_rank();
  Quad q;
  // both CTAs of a cluster decode the same cluster index: they leave together or not at all
  if (!decode_quad(p, blockIdx.x / 2, (int)rank, q)) return;
  const Unit& u = q.u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbar = smem_u32(smem + L::kBars);
#define bar(i) (sbar + 8u * (uint32_t)(i))
#define sQ(x) (sb + L::kQ + (uint32_t)(x) * kQBytes)
#define sKV(slot) (sb + L::kKV + (uint32_t)(slot) * kHalfBytes)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(bar(KV_FULL + i), 1);
      mbar_init(bar(KV_EMPTY + i), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(S_FULL + x), 1);
      mbar_init(bar(P_FULL + x), 8);  // the four warps of warpgroup x in each CTA
    }
    mbar_init(bar(Q_FULL), 1);
    mbar_init(bar(MMA_DONE), 1);
    mbar_init(bar(EXIT), 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialised before any arrival or load reaches them
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row_base = u.b * p.N;
  const bool leader = rank == 0;
  const uint32_t peer_abort = map_to(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Nothing is loaded for a cluster without a valid row: no MMA would consume the
    // loads, and a CTA must not retire with copies into its shared memory in flight.
    if (lane == 0 && u.kmax >= 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK64);
      prefetch_tmap(&tmV);
      const uint32_t q_full = map_to(bar(Q_FULL), 0);
      if (leader) {
        uint32_t qbytes = 0;  // every existing tile of the four is loaded by its CTA
        for (int x = 0; x < 2; ++x)
          for (int c = 0; c < 2; ++c) qbytes += (u.t[x] - (int)rank + c < u.ntiles) ? kQBytes : 0;
        mbar_arrive_expect_tx(bar(Q_FULL), qbytes);
      }
      for (int x = 0; x < 2; ++x) {
        if (u.t[x] >= u.ntiles) continue;
        const int row = row_base + tile_orig(p, u, u.t[x]);
        for (int c = 0; c < 2; ++c) tma_load_3d_pair(sQ(x) + c * kQChunk, &tmQ, c * 64, u.h, row, q_full);
      }
      int e = 0;
      bool ok = true;
      // one half tile per load: K rows [64·rank, +64) (both column chunks) or V columns [64·rank, +64)
      auto load = [&](bool isK, int k) {
        const int slot = e % kSlots;
        if (e >= kSlots) ok = s2_wait_cl(bar(KV_EMPTY + slot), ((e / kSlots) - 1) & 1, abort_flag, status, 1, peer_abort);
        if (!ok) return;
        if (leader) mbar_arrive_expect_tx(bar(KV_FULL + slot), 2 * kHalfBytes);
        const uint32_t full = map_to(bar(KV_FULL + slot), 0);
        const int row = row_base + tile_orig(p, u, k);
        if (isK) {
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(sKV(slot) + c * kKChunk, &tmK64, c * 64, u.h, row + 64 * (int)rank, full);
        } else {
          tma_load_3d_pair(sKV(slot), &tmV, 64 * (int)rank, u.h, row, full);
        }
        ++e;
      };
      // consumption order: K(k0), then per key tile V(k), K(next k)
      int kc = next_key(p, q, -1);
      if (kc >= 0) load(true, kc);
      while (ok && kc >= 0) {
        const int kn = next_key(p, q, kc);
        load(false, kc);
        if (!ok) break;
        if (kn >= 0) load(true, kn);
        kc = kn;
      }
      // every load of this CTA must land before the CTA retires: the last MMA_DONE
      // (waited below by every role) implies it
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && leader && u.kmax >= 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(256, 128, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(256, D, 0, 1);
#define ISSUE_QK(x, slot)                                                                         \
  do {                                                                                            \
    const uint64_t a0_ = umma_desc_sw128(sQ(x), 16, 1024), b0_ = umma_desc_sw128(sKV(slot), 16, 1024); \
    _Pragma("unroll") for (int kk = 0; kk < D / 16; ++kk) {                                       \
      const uint64_t offa_ = ((kk / 4) * kQChunk + (kk % 4) * 32) >> 4;                           \
      const uint64_t offb_ = ((kk / 4) * kKChunk + (kk % 4) * 32) >> 4;                           \
      umma_ss_pair(tmem + (x) * 128, a0_ + offa_, b0_ + offb_, idesc_qk, kk > 0);                 \
    }                                                                                             \
  } while (0)
#define ISSUE_PV(x, slot, acc)                                                                    \
  do {                                                                                            \
    const uint64_t b0_ = umma_desc_sw128(sKV(slot), kHalfBytes, 1024);                            \
    _Pragma("unroll") for (int kk = 0; kk < kTile / 16; ++kk) {                                   \
      umma_ts_pair(tmem + 256 + (x) * D, tmem + (x) * 128 + 8 * kk, b0_ + (uint64_t)(kk * 2048 >> 4), \
                   idesc_pv, ((acc) || kk > 0) ? 1u : 0u);                                        \
    }                                                                                             \
  } while (0)
      bool ok = s2_wait_cl(bar(Q_FULL), 0, abort_flag, status, 2, peer_abort);
      int npvA = 0, npvB = 0;
      int e = 0;
      int kc = next_key(p, q, -1);
      if (ok && kc >= 0) {
        const int eK = e++;
        ok = s2_wait_cl(bar(KV_FULL + eK % kSlots), (eK / kSlots) & 1, abort_flag, status, 2, peer_abort);
        tc_fence_after();
        if (ok && pair_takes(q, 0, kc)) {
          ISSUE_QK(0, eK % kSlots);
          umma_commit_pair(bar(S_FULL + 0));
        }
        if (ok && pair_takes(q, 1, kc)) {
          ISSUE_QK(1, eK % kSlots);
          umma_commit_pair(bar(S_FULL + 1));
        }
        umma_commit_pair(bar(KV_EMPTY + eK % kSlots));
      }
      int kn = kc >= 0 ? next_key(p, q, kc) : -1;
      int eV = e++;
      int eK = kn >= 0 ? e++ : -1;
      if (ok && kc >= 0) ok = s2_wait_cl(bar(KV_FULL + eV % kSlots), (eV / kSlots) & 1, abort_flag, status, 2, peer_abort);
      if (ok && kn >= 0) ok = s2_wait_cl(bar(KV_FULL + eK % kSlots), (eK / kSlots) & 1, abort_flag, status, 2, peer_abort);
      while (ok && kc >= 0) {
        const int sV = eV % kSlots, sK = eK >= 0 ? eK % kSlots : 0;
        if (pair_takes(q, 0, kc)) {
          ok = s2_wait_cl(bar(P_FULL + 0), npvA & 1, abort_flag, status, 2, peer_abort);
          if (!ok) break;
          tc_fence_after();
          ISSUE_PV(0, sV, npvA > 0);
          ++npvA;
        }
        if (kn >= 0 && pair_takes(q, 0, kn)) {
          ISSUE_QK(0, sK);
          umma_commit_pair(bar(S_FULL + 0));
        }
        const int knn = kn >= 0 ? next_key(p, q, kn) : -1;
        const int eV2 = kn >= 0 ? e++ : -1;
        const int eK2 = knn >= 0 ? e++ : -1;
        if (eV2 >= 0) ok = s2_wait_cl(bar(KV_FULL + eV2 % kSlots), (eV2 / kSlots) & 1, abort_flag, status, 2, peer_abort);
        if (ok && eK2 >= 0) ok = s2_wait_cl(bar(KV_FULL + eK2 % kSlots), (eK2 / kSlots) & 1, abort_flag, status, 2, peer_abort);
        if (!ok) break;
        if (pair_takes(q, 1, kc)) {
          ok = s2_wait_cl(bar(P_FULL + 1), npvB & 1, abort_flag, status, 2, peer_abort);
          if (!ok) break;
          tc_fence_after();
          ISSUE_PV(1, sV, npvB > 0);
          ++npvB;
        }
        if (kn >= 0 && pair_takes(q, 1, kn)) {
          ISSUE_QK(1, sK);
          umma_commit_pair(bar(S_FULL + 1));
        }
        umma_commit_pair(bar(KV_EMPTY + sV));
        if (kn >= 0) umma_commit_pair(bar(KV_EMPTY + sK));
        kc = kn;
        kn = knn;
        eV = eV2;
        eK = eK2;
      }
      // every issued MMA must be complete before either CTA reads or releases TMEM
      umma_commit_pair(bar(MMA_DONE));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups (both CTAs)
    const int x = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + x * 128;
    const uint32_t tO = tmem + lane_off + 256 + x * D;
    // scalars: indexing the unit's arrays with the runtime x would move them to local memory
    const int tx = x ? u.t[1] : u.t[0];
    const bool px = x ? q.own[1] : q.own[0];
    const bool pairx = x ? q.pair[1] : q.pair[0];
    const int kmaxx = x ? q.kmax[1] : q.kmax[0];
    const bool exists = tx < u.ntiles;
    const int q0 = exists ? tile_orig(p, u, tx) : 0;
    const bool row_valid = exists && (q0 + r) < p.n_valid;
    const uint32_t p_full = map_to(bar(P_FULL + x), 0);
    float m_used = -INFINITY, l = 0.f;
    int n = 0, nt = 0;  // key tiles of the pair / of them this tile takes
    bool ok = true;
    if (pairx) {
      for (int k = 0; k <= kmaxx && ok; ++k) {
        if (!ktile_valid(p, u, k)) continue;
        ok = s2_wait_cl(bar(S_FULL + x), n & 1, abort_flag, status, 4, peer_abort);
        if (!ok) break;
        tc_fence_after();
        uint32_t s[kTile];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld32(tS + j * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[j * 32]));
        tmem_wait_ld();
        // this tile takes key tile k only up to its own diagonal; beyond it (the
        // peer's diagonal) and for a tile without valid rows every column is masked
        const bool takes = px && k <= tx;
        const int cmax = takes ? col_limit(p, u, tx, k, r) : 0;
        nt += takes ? 1 : 0;
        if (!__all_sync(0xffffffffu, cmax == kTile)) {
#pragma unroll
          for (int c = 0; c < kTile; ++c)
            if (c >= cmax) s[c] = 0xff800000u;  // -inf
        }
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < kTile; c += 8) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq)
            mq[qq] = fmax3(mq[qq], __uint_as_float(s[c + 2 * qq]), __uint_as_float(s[c + 2 * qq + 1]));
        }
        const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * p.scale_log2;
        const float m_new = fmaxf(m_used, mx);
        const bool need = m_new > m_used + 8.0f;
        float factor = 1.f;
        if (need) {
          factor = ex2(m_used - m_new);
          l *= factor;
          m_used = m_new;
        }
        const float m_exp = (m_used == -INFINITY) ? 0.f : m_used;
        const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_exp, -m_exp);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < kTile; c += 2) {
          const float2 a = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), c2, nm2);
          const uint32_t pk = pack_bf16(ex2(a.x), ex2(a.y));
          s[c / 2] = pk;
          acc[(c / 2) & 3] =
              __fadd2_rn(acc[(c / 2) & 3], make_float2(__uint_as_float(pk << 16), __uint_as_float(pk & 0xffff0000u)));
        }
        const float2 acct = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l += acct.x + acct.y;
        // S_x(k) was issued behind O_x += P_x(k-1) V(k-1): O_x is complete here
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          const float f = need ? factor : 1.f;
#pragma unroll
          for (int j = 0; j < D / 32; ++j) {
            uint32_t o[32];
            tmem_ld32(tO + j * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
            tmem_st32(tO + j * 32, o);
          }
          tmem_wait_st();
        }
        tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&s[0]));
        tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&s[32]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(p_full);  // one arrival per warp: 8 per pair and tile
        ++n;
      }
    }
    // every MMA of the pair has completed (committed to both CTAs)
    if (ok && u.kmax >= 0) {
      ok = s2_wait_cl(bar(MMA_DONE), 0, abort_flag, status, 4, peer_abort);
      tc_fence_after();
    }
    // ---------------------------------------------------------- epilogue
    if (exists) {
      const bool have = px && ok && nt > 0;
      const float inv_l = (have && row_valid) ? 1.f / l : 0.f;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t o[32];
        if (have) {
          tmem_ld32(tO + j * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          const int col = j * 32 + pc * 8;
          const int chunk = col / 64, piece = (col % 64) / 8;
          const uint32_t addr = sQ(x) + chunk * kQChunk + r * 128 + ((piece ^ (r & 7)) << 4);
          const uint32_t* oo = &o[pc * 8];
          st_shared_v4(addr, pack_bf16(__uint_as_float(oo[0]) * inv_l, __uint_as_float(oo[1]) * inv_l),
                       pack_bf16(__uint_as_float(oo[2]) * inv_l, __uint_as_float(oo[3]) * inv_l),
                       pack_bf16(__uint_as_float(oo[4]) * inv_l, __uint_as_float(oo[5]) * inv_l),
                       pack_bf16(__uint_as_float(oo[6]) * inv_l, __uint_as_float(oo[7]) * inv_l));
        }
      }
      const float lse_v = (have && row_valid) ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      lse[((size_t)u.b * p.H + u.h) * p.N + q0 + r] = lse_v;
      fence_proxy_async_smem();
      named_bar_sync(1 + x, 128);
      if (r == 0) {
        for (int c = 0; c < 2; ++c) tma_store_3d(&tmO, sQ(x) + c * kQChunk, c * 64, u.h, row_base + q0);
        tma_store_commit();
        tma_store_wait_all();
      }
    }
  }

  // Both CTAs have finished with tensor memory (their epilogues' loads are
  // complete) before the paired allocation is released.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(map_to(bar(EXIT), rank ^ 1u));
    wait_exit(bar(EXIT), status);
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
#undef ISSUE_QK
#undef ISSUE_PV
#undef bar
#undef sQ
#undef sKV
}

int launch_fwd_pair(const FwdArgs& a) {
  using L = fwd2::Layout;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(s2_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return (int)e;
  const int clusters = groups_of(a.plan.B * a.plan.H, a.plan.hg_fwd) * a.plan.hg_fwd * a.plan.quad_ranks;
  s2_fwd_pair_kernel<<<2 * clusters, fwd2::kThreads, L::kAlloc, a.stream>>>(*a.tmQ, *a.tmK64, *a.tmV, *a.tmO, a.plan,
                                                                           a.lse, a.status);
  return (int)cudaGetLastError();
}

}  // namespace s2
