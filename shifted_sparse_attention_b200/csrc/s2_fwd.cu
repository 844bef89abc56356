// s2_fwd.cu -- S²-Attn forward on sm_100a (tcgen05 tensor cores, TMA, TMEM).
//
// Computes, per head and query row i with visible set S_i
// ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调", §3):
//     o_i = sum_{j in S_i} softmax_j(q_i·k_j / sqrt(D)) v_j,
//     lse_i = ln sum_{j in S_i} exp(q_i·k_j / sqrt(D)),
// where S_i is the causal part of i's group (§1, see s2_index.cuh).
// Only key tiles of i's own segment up to the diagonal are visited: no
// off-group tile is ever loaded or multiplied, so the work is O(N·G).
//
// CTA = two consecutive 128-row query tiles (A, B) of one segment sharing
// every K/V tile.  Warp roles (320 threads):
//   warps 0-3  softmax of tile A (thread = one query row = one TMEM lane)
//   warps 4-7  softmax of tile B
//   warp  8    TMA producer: Q tiles once, then the K/V stream
//   warp  9    TMEM allocator and tcgen05.mma issuer (one thread)
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A and O_B at 256 + x·D.
// The softmax writes P (bf16 pairs) over the first 64 columns of its S, and
// O += P V reads it from there as the A operand: P never touches shared
// memory, whose bandwidth the score MMAs (both operands in shared memory)
// already use in full.  Shared memory: Q_A, Q_B and a ring of five K/V slots;
// all tiles are 128-byte-swizzled, 1024-byte aligned, as TMA writes and UMMA
// reads them.  MMA order per key tile k:
//     O_A += P_A(k) V(k), S_A(k+1) = Q_A K(k+1)^T, O_B += P_B(k) V(k), S_B(k+1)
// so each softmax warpgroup works on its tile while the tensor core runs the
// other tile's two products, and S_x(k+1) overwrites P_x(k) only behind the
// MMA that reads it.
// Softmax uses base-2 exponentials with a lazily updated running max: O and
// l are rescaled only when the row max grows by more than 8 (a factor 256),
// which keeps bf16 P and fp32 sums exact enough and skips most rescales.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_debug.cuh"
#include "s2_index.cuh"
#include "s2_kernels.h"
#include "sm100_ptx.cuh"

namespace s2 {

namespace fwd {

constexpr int kThreads = 320;
constexpr int kSlots = 5;
constexpr int kChunkBytes = kTile * 64 * 2;  // 128 rows x 64 bf16 = one 128B-swizzle column block

enum Bar {
  KV_FULL = 0,      // + slot (5)
  KV_EMPTY = 5,     // + slot (5)
  S_FULL = 10,      // + tile (2)
  P_FULL = 12,      // + tile (2)
  Q_FULL = 14,
  MMA_DONE = 15,
  NUM_BARS = 16
};

template <int D>
struct Layout {
  static constexpr int kQBytes = kTile * D * 2;
  static constexpr int kKVBytes = kTile * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kKV = 2 * kQBytes;
  static constexpr int kBars = kKV + kSlots * kKVBytes;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// Query tile x (its index tx, whether it holds a valid row px, and the span
// [lo, hi) of the documents touching it) takes part at key tile k.
// Without documents (kDocs false) the span test is skipped outright: it costs
// the single MMA-issuing thread a tile-origin computation per key tile.
template <bool kDocs>
__device__ __forceinline__ bool takes(const Plan& p, const Unit& u, bool px, int tx, int lo, int hi, int k) {
  if constexpr (kDocs) return px && k <= tx && tile_meets(tile_orig(p, u, k), lo, hi);
  return px && k <= tx;
}

// Smallest key tile > k that holds a valid key and that one of the unit's two
// query tiles takes part at, or -1.
template <bool kDocs>
__device__ __forceinline__ int next_k(const Plan& p, const Unit& u, int k, bool pA, int tA, int lA, int hA, bool pB,
                                      int tB, int lB, int hB) {
  for (int j = k + 1; j <= u.kmax; ++j)
    if (ktile_valid(p, u, j) &&
        (takes<kDocs>(p, u, pA, tA, lA, hA, j) || takes<kDocs>(p, u, pB, tB, lB, hB, j)))
      return j;
  return -1;
}

}  // namespace fwd

// kDocs: a document mask is present (p.docs != nullptr).  Without it the
// document tests fold away at compile time.
template <int D, bool kDocs>
__global__ void __launch_bounds__(fwd::kThreads, 1)
    s2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ Plan plan, float* __restrict__ lse, int* __restrict__ status) {
  using namespace fwd;
  const Plan& p = plan;
  using L = Layout<D>;
  constexpr int kChunks = D / 64;

  Unit u;
  if (!decode_unit(p, blockIdx.x, u)) return;
  // The two query tiles as scalars: indexing u.t[] / u.part[] with a runtime
  // tile number would put the whole struct in local memory.
  const int tA = u.t[0], tB = u.t[1];
  const bool pA = u.part[0], pB = u.part[1];
  // spans of the documents touching each query tile (everything without documents)
  int lA = 0, hA = p.N, lB = 0, hB = p.N;
  if (kDocs && pA) doc_span(p, u.b, tile_orig(p, u, tA), lA, hA);
  if (kDocs && pB) doc_span(p, u.b, tile_orig(p, u, tB), lB, hB);
#define NEXT_K(k) next_k<kDocs>(p, u, (k), pA, tA, lA, hA, pB, tB, lB, hB)
#define TAKES_A(k) takes<kDocs>(p, u, pA, tA, lA, hA, (k))
#define TAKES_B(k) takes<kDocs>(p, u, pB, tB, lB, hB, (k))

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // Addresses are plain values (macros, #undef'd after the kernel): no lambda
  // captures, so nothing the MMA issuer needs lives in memory.
  const uint32_t sbar = smem_u32(bars);
#define bar(i) (sbar + 8u * (uint32_t)(i))
#define sQ(x) (sb + L::kQ + (uint32_t)(x) * L::kQBytes)
#define sKV(slot) (sb + L::kKV + (uint32_t)(slot) * L::kKVBytes)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(bar(KV_FULL + i), 1);
      mbar_init(bar(KV_EMPTY + i), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(S_FULL + x), 1);
      mbar_init(bar(P_FULL + x), 128);
    }
    mbar_init(bar(Q_FULL), 1);
    mbar_init(bar(MMA_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row_base = u.b * p.N;  // TMA outer coordinate of position 0 of this batch row

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && u.kmax >= 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      uint32_t qbytes = 0;
      qbytes += pA ? L::kQBytes : 0;
      qbytes += pB ? L::kQBytes : 0;
      mbar_arrive_expect_tx(bar(Q_FULL), qbytes);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (!(x ? pB : pA)) continue;
        const int x0 = tile_orig(p, u, x ? tB : tA);
        const int row = row_base + x0;
        if (!(S2_IN(kSiteFwdQ, x0, p.q_begin, p.n_valid) && S2_IN(kSiteFwdQ, x0, 0, p.N - kTile + 1) &&
              S2_IN(kSiteFwdQ, row, 0, (long long)p.B * p.N - kTile + 1))) {
          *abort_flag = 1;  // the debug build skips the access and gives up
          continue;
        }
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(sQ(x) + c * kChunkBytes, &tmQ, c * 64, u.h, row, bar(Q_FULL));
      }
      int e = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* tm, int k) {
        const int slot = e % kSlots;
        if (e >= kSlots) ok = s2_wait(bar(KV_EMPTY + slot), ((e / kSlots) - 1) & 1, abort_flag, status, 1);
        if (!ok) return;
        mbar_arrive_expect_tx(bar(KV_FULL + slot), L::kKVBytes);
        const int x0 = tile_orig(p, u, k);
        const int row = row_base + x0;
        if (S2_IN(kSiteFwdKV, x0, p.k_begin, p.n_valid) && S2_IN(kSiteFwdKV, x0, 0, p.N - kTile + 1) &&
            S2_IN(kSiteFwdKV, row, 0, (long long)p.B * p.N - kTile + 1)) {
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(sKV(slot) + c * kChunkBytes, tm, c * 64, u.h, row, bar(KV_FULL + slot));
        } else {
          *abort_flag = 1;
        }
        ++e;
      };
      // consumption order: K(k0), then per key tile V(k), K(next k)
      int kc = NEXT_K(-1);
      if (kc >= 0) load(&tmK, kc);
      while (ok && kc >= 0) {
        const int kn = NEXT_K(kc);
        load(&tmV, kc);
        if (!ok) break;
        if (kn >= 0) load(&tmK, kn);
        kc = kn;
      }
      // drain: the last loads must land before the CTA retires (also after an abort)
      for (int d = (e > kSlots ? e - kSlots : 0); d < e; ++d)
        s2_wait_drain(bar(KV_FULL + d % kSlots), (d / kSlots) & 1, status, 1);
      s2_wait_drain(bar(Q_FULL), 0, status, 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && u.kmax >= 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, D, 0, 1);
      // Descriptors are built once per group and advanced by compile-time
      // offsets (in 16-byte units): issuing an MMA then costs a 64-bit add.
#define ISSUE_QK(x, slot)                                                                         \
  do {                                                                                            \
    const uint64_t a0_ = umma_desc_sw128(sQ(x), 16, 1024), b0_ = umma_desc_sw128(sKV(slot), 16, 1024); \
    _Pragma("unroll") for (int kk = 0; kk < D / 16; ++kk) {                                       \
      const uint64_t off_ = ((kk / 4) * kChunkBytes + (kk % 4) * 32) >> 4;                        \
      umma_ss(tmem + (x) * 128, a0_ + off_, b0_ + off_, idesc_qk, kk > 0);                         \
    }                                                                                             \
  } while (0)
#define ISSUE_PV(x, slot, acc)                                                                    \
  do {                                                                                            \
    const uint64_t b0_ = umma_desc_sw128(sKV(slot), kChunkBytes, 1024);                           \
    _Pragma("unroll") for (int kk = 0; kk < kTile / 16; ++kk) {                                   \
      umma_ts(tmem + 256 + (x) * D, tmem + (x) * 128 + 8 * kk, b0_ + (uint64_t)(kk * 2048 >> 4),   \
              idesc_pv, ((acc) || kk > 0) ? 1u : 0u);                                             \
    }                                                                                             \
  } while (0)
      bool ok = s2_wait(bar(Q_FULL), 0, abort_flag, status, 2);
      int npvA = 0, npvB = 0;
      int e = 0;  // position in the K/V load sequence
      int kc = NEXT_K(-1);
      if (ok && kc >= 0) {
        const int eK = e++;
        ok = s2_wait(bar(KV_FULL + eK % kSlots), (eK / kSlots) & 1, abort_flag, status, 2);
        if (ok && TAKES_A(kc)) {
          ISSUE_QK(0, eK % kSlots);
          umma_commit(bar(S_FULL + 0));
        }
        if (ok && TAKES_B(kc)) {
          ISSUE_QK(1, eK % kSlots);
          umma_commit(bar(S_FULL + 1));
        }
        umma_commit(bar(KV_EMPTY + eK % kSlots));
      }
      // loads of the first iteration: V(kc) and K(next)
      int kn = kc >= 0 ? NEXT_K(kc) : -1;
      int eV = e++;
      int eK = kn >= 0 ? e++ : -1;
      if (ok && kc >= 0) ok = s2_wait(bar(KV_FULL + eV % kSlots), (eV / kSlots) & 1, abort_flag, status, 2);
      if (ok && kn >= 0) ok = s2_wait(bar(KV_FULL + eK % kSlots), (eK / kSlots) & 1, abort_flag, status, 2);
      while (ok && kc >= 0) {
        // per tile: O_x += P_x(kc) V(kc), then S_x(kn) into the same TMEM columns
        const int sV = eV % kSlots, sK = eK % kSlots;
        // (a tile's key tiles need not start together with the other tile's under a
        // document mask: S_x(kn) is issued whenever x takes kn, behind any O_x += P_x V)
        if (TAKES_A(kc)) {
          ok = s2_wait(bar(P_FULL + 0), npvA & 1, abort_flag, status, 2);
          if (!ok) break;
          tc_fence_after();
          ISSUE_PV(0, sV, npvA > 0);
          ++npvA;
        }
        if (kn >= 0 && TAKES_A(kn)) {
          ISSUE_QK(0, sK);
          umma_commit(bar(S_FULL + 0));
        }
        // The next iteration's tile and loads, while tile A's products are queued:
        // the issuing thread's bookkeeping then never leaves the tensor core idle.
        const int knn = kn >= 0 ? NEXT_K(kn) : -1;
        const int eV2 = kn >= 0 ? e++ : -1;   // V(kn)
        const int eK2 = knn >= 0 ? e++ : -1;  // K(knn)
        if (eV2 >= 0) ok = s2_wait(bar(KV_FULL + eV2 % kSlots), (eV2 / kSlots) & 1, abort_flag, status, 2);
        if (ok && eK2 >= 0) ok = s2_wait(bar(KV_FULL + eK2 % kSlots), (eK2 / kSlots) & 1, abort_flag, status, 2);
        if (!ok) break;
        if (TAKES_B(kc)) {
          ok = s2_wait(bar(P_FULL + 1), npvB & 1, abort_flag, status, 2);
          if (!ok) break;
          tc_fence_after();
          ISSUE_PV(1, sV, npvB > 0);
          ++npvB;
        }
        if (kn >= 0 && TAKES_B(kn)) {
          ISSUE_QK(1, sK);
          umma_commit(bar(S_FULL + 1));
        }
        umma_commit(bar(KV_EMPTY + sV));
        if (kn >= 0) umma_commit(bar(KV_EMPTY + sK));
        kc = kn;
        kn = knn;
        eV = eV2;
        eK = eK2;
      }
      // every issued MMA must be complete before TMEM is released (also after an abort)
      umma_commit(bar(MMA_DONE));
      s2_wait_drain(bar(MMA_DONE), 0, status, 2);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warpgroups
    const int x = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + x * 128;
    const uint32_t tO = tmem + lane_off + 256 + x * D;
    const int tx = x ? tB : tA;
    const bool px = x ? pB : pA;
    const int lx = x ? lB : lA, hx = x ? hB : hA;
    // S_x and O_x within the 512 allocated columns
    if (!(S2_IN(kSiteFwdTmem, x * 128 + 128, 1, 257) && S2_IN(kSiteFwdTmem, 256 + x * D + D, 257, 513)))
      *abort_flag = 1;
    if (tx >= 0) {
      const int q0 = tile_orig(p, u, tx);
      const bool row_valid = (q0 + r) < p.n_valid;
      float m_used = -INFINITY, l = 0.f;
      int n = 0;
      bool ok = true;
      if (px) {
        for (int k = 0; k <= tx && ok; ++k) {
          if (!ktile_valid(p, u, k) || (kDocs && !tile_meets(tile_orig(p, u, k), lx, hx))) continue;
          ok = s2_wait(bar(S_FULL + x), n & 1, abort_flag, status, 4);
          if (!ok) break;
          tc_fence_after();
          uint32_t s[kTile];
          tmem_ld128(tS, s);
          tmem_wait_ld();

          // Masks (the causal triangle of the diagonal tile, padded keys or rows,
          // the row's document) only where some row of the warp needs them.
          int cmin = 0, cmax;
          if constexpr (kDocs)
            row_cols(p, u, tx, k, r, cmin, cmax);
          else
            cmax = col_limit(p, u, tx, k, r);
          if (!__all_sync(0xffffffffu, cmin == 0 && cmax == kTile)) {
#pragma unroll
            for (int c = 0; c < kTile; ++c)
              if (c < cmin || c >= cmax) s[c] = 0xff800000u;  // -inf
          }
          // Row max as a 4-way tree of 3-input max (short dependency chains), then
          // scaled once (scale > 0 keeps the order).
          float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < kTile; c += 8) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mq[q] = fmax3(mq[q], __uint_as_float(s[c + 2 * q]), __uint_as_float(s[c + 2 * q + 1]));
          }
          const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * p.scale_log2;
          const float m_new = fmaxf(m_used, mx);
          const bool need = m_new > m_used + 8.0f;
          float factor = 1.f;
          if (need) {
            factor = ex2(m_used - m_new);  // 0 when m_used = -inf
            l *= factor;
            m_used = m_new;
          }
          const float m_exp = (m_used == -INFINITY) ? 0.f : m_used;
          // p = 2^(x·c - m) two columns at a time, rounded to bf16 pairs in place
          // (s[c/2] <- pair c, c+1); l sums the ROUNDED weights in four packed
          // accumulators, so o = sum p~ v / sum p~ stays a convex combination of the v_j.
          const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 nm2 = make_float2(-m_exp, -m_exp);
          float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < kTile; c += 2) {
            const float2 a = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), c2, nm2);
            const uint32_t pk = pack_bf16(ex2(a.x), ex2(a.y));
            s[c / 2] = pk;
            acc[(c / 2) & 3] = __fadd2_rn(acc[(c / 2) & 3], make_float2(__uint_as_float(pk << 16), __uint_as_float(pk & 0xffff0000u)));
          }
          const float2 acc01 = __fadd2_rn(acc[0], acc[1]), acc23 = __fadd2_rn(acc[2], acc[3]);
          const float2 acct = __fadd2_rn(acc01, acc23);
          l += acct.x + acct.y;

          // S_x(k) was issued behind O_x += P_x(k-1) V(k-1), so O_x is complete here
          if (n > 0) {
            if (__any_sync(0xffffffffu, need)) {
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
          }
          // P (bf16 pairs) -> TMEM columns [0, 64) of S_x, the A operand of O_x += P_x V
          tmem_st64(tS, *reinterpret_cast<const uint32_t(*)[64]>(&s[0]));
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(P_FULL + x));
          ++n;
        }
        if (ok && n > 0) {  // the last O_x += P_x V has completed
          ok = s2_wait(bar(MMA_DONE), 0, abort_flag, status, 4);
          tc_fence_after();
        }
      }
      // ---------------------------------------------------------- epilogue
      const bool have = px && ok && n > 0;
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
          const int col = j * 32 + pc * 8;  // first of 8 columns
          const int chunk = col / 64, piece = (col % 64) / 8;
          const uint32_t addr = sQ(x) + chunk * kChunkBytes + r * 128 + ((piece ^ (r & 7)) << 4);
          const uint32_t* oo = &o[pc * 8];
          st_shared_v4(addr, pack_bf16(__uint_as_float(oo[0]) * inv_l, __uint_as_float(oo[1]) * inv_l),
                       pack_bf16(__uint_as_float(oo[2]) * inv_l, __uint_as_float(oo[3]) * inv_l),
                       pack_bf16(__uint_as_float(oo[4]) * inv_l, __uint_as_float(oo[5]) * inv_l),
                       pack_bf16(__uint_as_float(oo[6]) * inv_l, __uint_as_float(oo[7]) * inv_l));
        }
      }
      const float lse_v = (have && row_valid) ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t lse_at = ((size_t)u.b * p.H + u.h) * p.N + q0 + r;
      if (S2_IN(kSiteFwdOut, lse_at, 0, (long long)p.B * p.H * p.N)) lse[lse_at] = lse_v;
      const bool out_in = S2_IN(kSiteFwdOut, q0, 0, p.N - kTile + 1);
      fence_proxy_async_smem();
      named_bar_sync(1 + x, 128);
      if (r == 0 && out_in) {
        for (int c = 0; c < kChunks; ++c)
          tma_store_3d(&tmO, sQ(x) + c * kChunkBytes, c * 64, u.h, row_base + q0);
        tma_store_commit();
        tma_store_wait_all();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

#undef ISSUE_QK
#undef ISSUE_PV
#undef NEXT_K
#undef TAKES_A
#undef TAKES_B
#undef bar
#undef sQ
#undef sKV

template <int D, bool kDocs>
int launch_fwd_impl(const FwdArgs& a) {
  using L = fwd::Layout<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e =
      cudaFuncSetAttribute(s2_fwd_kernel<D, kDocs>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return (int)e;
  const int grid = grid_fwd(a.plan);
  s2_fwd_kernel<D, kDocs><<<grid, fwd::kThreads, L::kAlloc, a.stream>>>(*a.tmQ, *a.tmK, *a.tmV, *a.tmO, a.plan,
                                                                        a.lse, a.status);
  return (int)cudaGetLastError();
}

int launch_fwd(const FwdArgs& a) {
  const bool docs = a.plan.docs != nullptr;
  if (a.plan.D == 64) return docs ? launch_fwd_impl<64, true>(a) : launch_fwd_impl<64, false>(a);
  return docs ? launch_fwd_impl<128, true>(a) : launch_fwd_impl<128, false>(a);
}

}  // namespace s2
