// s2_bwd.cu -- S²-Attn backward on sm_100a (tcgen05 tensor cores, TMA, TMEM).
//
// Gradients of L = sum_i dout_i·o_i over the same visible sets as the
// forward ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调", §3: with
// a_ij = exp(scale q_i·k_j - lse_i) and g_i = dout_i,
//     dL/dz_ij = a_ij (g_i·v_j - Delta_i),  Delta_i = g_i·o_i,
//     dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i a_ij g_i).
// Only in-group pairs are ever computed (§1: the backward stays sparse; the
// shift and reshape only permute gradients, which here is index math).
//
// Three launches on the caller's stream:
//   1. s2_bwd_pre: -Delta_i = -(dout_i·o_i) and -lse_i·log2(e) (-inf on
//      padded rows, which zeroes their probabilities), per [B, H, N].
//   2. s2_bwd_dkdv_kernel: key-major, one CTA per 128-key tile of a segment,
//      walking the query tiles from the diagonal to the segment's end:
//        S^T = K Q^T, dP^T = V dO^T (TMEM);  P^T = exp2(S^T·c - lse2) and
//        dS^T = P^T (dP^T - Delta) on the CUDA cores, both written back to
//        TMEM as bf16;  dV += P^T dO and dK += dS^T Q with A read from TMEM.
//   3. the dq pass, query-major, one CTA per 128-query tile, walking the key
//      tiles from the segment start to the diagonal, in one of two forms:
//      - s2_bwd_dq_ds_kernel (stages with S2_BWD_STORE_DS): the dK/dV pass
//        has also written every dS tile (bf16) to the workspace, and
//        dQ += dS K streams them back (HBM-bound, no exponentials);
//      - s2_bwd_dq_kernel: recomputes S = Q K^T and dP = dO V^T (TMEM),
//        dS = P (dP - Delta) -> TMEM (bf16), dQ += dS K with A from TMEM.
//      Either way dq = bf16(dQ / sqrt(D)) is written once.
// The recomputing form does 7 instead of 5 tile products per (key tile,
// query tile) pair; the stored form trades the two extra products for 32 KB
// of dS written and read per pair.  Neither needs a float32 dq accumulator:
// a fused kernel adds one float32 partial of every dq row per key tile into
// global memory, and the L2's float32 reduction rate (a few TB/s) then bounds
// the whole backward.  dq is also bitwise deterministic this way.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_debug.cuh"
#include "s2_index.cuh"
#include "s2_kernels.h"
#include "sm100_ptx.cuh"

namespace s2 {

namespace bwd {

constexpr int kThreads = 320;  // warps 0-7 elementwise, 8 TMA producer, 9 TMEM + MMA issuer
constexpr int kChunkBytes = kTile * 64 * 2;  // 128 rows x 64 bf16: one 128-byte-swizzle column block

// Descriptor offsets (16-byte units) of MMA K-step kk over a 128-byte-swizzled
// tile: K-major operands step 32 bytes inside a 64-column chunk, then a chunk;
// MN-major operands step 16 rows.
#define S2_KM_OFF(kk) ((uint64_t)((((kk) / 4) * kChunkBytes + ((kk) % 4) * 32) >> 4))
#define S2_MN_OFF(kk) ((uint64_t)(((kk) * 2048) >> 4))

// Next query tile after qt (up to the segment end) that holds a valid row and
// meets the span [lo, hi) of the documents touching the key tile, or -1.
__device__ __forceinline__ int next_q(const Plan& p, const Unit& u, int qt, int lo, int hi) {
  for (int j = qt + 1; j <= u.kmax; ++j)
    if (qtile_valid(p, u, j) && tile_meets(tile_orig(p, u, j), lo, hi)) return j;
  return -1;
}

// Next valid key tile after k (up to the query tile u.t[0]) that meets the
// span [lo, hi) of the documents touching the query tile, or -1.
__device__ __forceinline__ int next_k(const Plan& p, const Unit& u, int k, int lo, int hi) {
  for (int j = k + 1; j <= u.t[0]; ++j)
    if (ktile_valid(p, u, j) && tile_meets(tile_orig(p, u, j), lo, hi)) return j;
  return -1;
}

// An accumulator (TMEM, lane = row) -> bf16 -> shared staging laid out as
// two 128-byte-swizzled chunks of 64 columns; warpgroup x converts columns
// [x·D/2, x·D/2 + D/2) of its row.  Rows that are not valid are written as 0.
template <int D>
__device__ __forceinline__ void acc_to_smem(uint32_t tacc, uint32_t lane_off, int x, int row, bool have,
                                            bool row_valid, float mul, uint32_t stage) {
#pragma unroll
  for (int c2 = 0; c2 < D / 64; ++c2) {
    const int d0 = x * (D / 2) + 32 * c2;
    uint32_t v[32];
    if (have) {
      tmem_ld32(tacc + lane_off + d0, v);
      tmem_wait_ld();
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = d0 + 8 * q;
      const int chunk = col / 64, piece = (col % 64) / 8;
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float a = (have && row_valid) ? __uint_as_float(v[8 * q + 2 * t]) * mul : 0.f;
        const float b = (have && row_valid) ? __uint_as_float(v[8 * q + 2 * t + 1]) * mul : 0.f;
        w[t] = pack_bf16(a, b);
      }
      st_shared_v4(stage + chunk * kChunkBytes + row * 128 + ((piece ^ (row & 7)) << 4), w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace bwd

// ------------------------------------------------------------------ preprocess
// kTpr = D/8 threads per (b, i, h) row, 8 bf16 (16 bytes) each.  Stores the
// negated statistics the passes add: -Delta = -(dout·o) and -lse·log2(e)
// (-inf on padded rows, which zeroes their probabilities).
template <int D>
__global__ void __launch_bounds__(256) s2_bwd_pre(const __nv_bfloat16* __restrict__ o,
                                                   const __nv_bfloat16* __restrict__ dout,
                                                   const float* __restrict__ lse, float* __restrict__ delta,
                                                   float* __restrict__ lse2, int B, int N, int H, int q_begin,
                                                   int n_valid) {
  constexpr int kTpr = D / 8;
  constexpr int kRowsPerBlock = 256 / kTpr;
  const long long row = (long long)blockIdx.x * kRowsPerBlock + threadIdx.x / kTpr;
  const int sub = threadIdx.x % kTpr;
  const long long rows = (long long)B * N * H;
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + sub * 8);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + row * D + sub * 8);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 fa = __bfloat1622float2(a2[t]), fg = __bfloat1622float2(g2[t]);
      acc = fmaf(fa.x, fg.x, acc);
      acc = fmaf(fa.y, fg.y, acc);
    }
  }
#pragma unroll
  for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, kTpr);
  if (row < rows && sub == 0) {
    const int h = (int)(row % H);
    const long long bi = row / H;
    const int i = (int)(bi % N), b = (int)(bi / N);
    const size_t at = ((size_t)b * H + h) * N + i;
    const bool valid = i >= q_begin && i < n_valid;
    delta[at] = valid ? -acc : 0.f;
    lse2[at] = valid ? -lse[at] * 1.4426950408889634f : -INFINITY;
  }
}

// ------------------------------------------------------------------ dK, dV pass
// Tensor memory (512 columns): R1 [0, 128) S^T then P^T; R2 [128, 256) dP^T
// then dS^T; dV [256, 256 + D); dK [256 + D, 256 + 2D).  P^T and dS^T are
// bf16 pairs: query columns [64x, 64x + 64) of a tile land in columns
// [64x, 64x + 32) of their region, which warpgroup x has already read.
// Issue order per query tile n (one thread of warp 9):
//   dP(n) -> R2    (behind dK(n-1), the last reader of dS^T(n-1))
//   dV(n)          once P^T(n) is in R1
//   S(n+1) -> R1   (behind dV(n), the last reader of P^T(n))
//   dK(n)          once dS^T(n) is in R2
// so the exponentials of tile n+1 overlap dK(n) and dP(n+1), and dS(n)
// overlaps dV(n) and S(n+1).  Elementwise thread = key row j (TMEM lane),
// warpgroup x = query columns [64x, 64x + 64); order P(0), [dS(n), P(n+1)].
// Q tiles (with their -lse2 rows) live in a ring of three slots, dO tiles
// (with their -Delta rows) in a ring of two: a slot is refilled as soon as
// its last reader is done (dK for Q; dV and the dS step for dO), which puts
// about six tile products between a load and its first use -- the L2's
// latency under full load is of that order.
namespace dkdv {

constexpr int kQSlots = 3, kOSlots = 2;
enum Bar {
  KV_FULL = 0,
  Q_FULL = 1,    // + slot (3)
  Q_EMPTY = 4,   // + slot (3)
  O_FULL = 7,    // + slot (2)
  O_EMPTY = 9,   // + slot (2): dV's commit + the 256 elementwise threads after their dS step
  S_FULL = 11,
  DP_FULL = 12,
  P_READY = 13,
  DS_READY = 14,
  ACC_DONE = 15,
  NUM_BARS = 16
};

template <int D>
struct Layout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kRowBytes = kTile * 4;  // one float32 statistic of a query tile
  static constexpr int kK = 0;
  static constexpr int kV = kTileBytes;
  static constexpr int kQ = 2 * kTileBytes;                  // + slot * kTileBytes
  static constexpr int kdO = kQ + kQSlots * kTileBytes;      // + slot * kTileBytes
  static constexpr int kLse = kdO + kOSlots * kTileBytes;    // -lse2 rows, + slot * kRowBytes
  static constexpr int kDelta = kLse + kQSlots * kRowBytes;  // -Delta rows, + slot * kRowBytes
  static constexpr int kBars = kDelta + kOSlots * kRowBytes;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
};

}  // namespace dkdv

// kStoreDS: also write every dS tile (bf16, key rows x query columns) to
// `ds_store` for the stored-dS dQ pass.
template <int D, bool kStoreDS>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    s2_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                       const __grid_constant__ Plan p, const float* __restrict__ delta,
                       const float* __restrict__ lse2, __nv_bfloat16* __restrict__ ds_store,
                       int* __restrict__ status) {
  using namespace bwd;
  using namespace dkdv;
  using L = dkdv::Layout<D>;
  constexpr int kChunks = D / 64;

  Unit u;
  if (!decode_kv_unit(p, blockIdx.x, u)) return;
  extern __shared__ __align__(1024) uint8_t smem_kv[];
  // 128-byte swizzle atoms need a 1024-byte aligned base; report and leave otherwise.
  if (smem_u32(smem_kv) & 1023u) {
    if (threadIdx.x == 0) atomicOr(status, 256);
    return;
  }
  const int kt = u.t[0];
  const int k0 = tile_orig(p, u, kt);
  int lK, hK;  // span of the documents touching the key tile
  doc_span(p, u.b, k0, lK, hK);
  // first query tile: the diagonal, unless it lies in a sequence-parallel halo
  // (rows that are keys only); a key tile no query reaches gets dK = dV = 0
  const int q_first = !u.part[0] ? -1 : qtile_valid(p, u, kt) ? kt : next_q(p, u, kt, lK, hK);
  const bool kvalid = q_first >= 0;

  uint8_t* smem = smem_kv;
  const uint32_t sb = smem_u32(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbar = sb + L::kBars;
#define bar(i) (sbar + 8u * (uint32_t)(i))
#define sQ(st) (sb + L::kQ + (uint32_t)(st) * L::kTileBytes)
#define sdO(st) (sb + L::kdO + (uint32_t)(st) * L::kTileBytes)
  const uint32_t sK = sb + L::kK, sV = sb + L::kV;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar(KV_FULL), 1);
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(bar(Q_FULL + i), 1);
      mbar_init(bar(Q_EMPTY + i), 1);
    }
    for (int i = 0; i < kOSlots; ++i) {
      mbar_init(bar(O_FULL + i), 1);
      mbar_init(bar(O_EMPTY + i), 1 + 256);
    }
    mbar_init(bar(S_FULL), 1);
    mbar_init(bar(DP_FULL), 1);
    mbar_init(bar(P_READY), 256);
    mbar_init(bar(DS_READY), 256);
    mbar_init(bar(ACC_DONE), 1);
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
  const uint32_t tR1 = tmem, tR2 = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const int row_base = u.b * p.N;
  const size_t stat_base = ((size_t)u.b * p.H + u.h) * p.N;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && kvalid) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(KV_FULL), 2 * L::kTileBytes);
      if (S2_IN(kSiteKvK, k0, p.k_begin, p.n_valid) && S2_IN(kSiteKvK, k0, 0, p.N - kTile + 1) &&
          S2_IN(kSiteKvK, row_base + k0, 0, (long long)p.B * p.N - kTile + 1)) {
        for (int c = 0; c < kChunks; ++c) {
          tma_load_3d(sK + c * kChunkBytes, &tmK, c * 64, u.h, row_base + k0, bar(KV_FULL));
          tma_load_3d(sV + c * kChunkBytes, &tmV, c * 64, u.h, row_base + k0, bar(KV_FULL));
        }
      } else {
        *abort_flag = 1;  // the debug build skips the access and gives up
      }
      int n = 0;
      bool ok = true;
      for (int qt = q_first; ok && qt >= 0; qt = next_q(p, u, qt, lK, hK)) {
        const int q0 = tile_orig(p, u, qt);
        const int sq = n % kQSlots, so = n % kOSlots;
        if (!(S2_IN(kSiteKvQ, q0, p.q_begin, p.n_valid) && S2_IN(kSiteKvQ, q0, 0, p.N - kTile + 1) &&
              S2_IN(kSiteKvQ, row_base + q0, 0, (long long)p.B * p.N - kTile + 1) &&
              S2_IN(kSiteKvQ, stat_base + q0, 0, (long long)p.B * p.H * p.N - kTile + 1))) {
          *abort_flag = 1;
          break;
        }
        if (n >= kQSlots) ok = s2_wait(bar(Q_EMPTY + sq), ((n / kQSlots) - 1) & 1, abort_flag, status, 8);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(Q_FULL + sq), L::kTileBytes + L::kRowBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(sQ(sq) + c * kChunkBytes, &tmQ, c * 64, u.h, row_base + q0, bar(Q_FULL + sq));
        bulk_load(sb + L::kLse + sq * L::kRowBytes, lse2 + stat_base + q0, L::kRowBytes, bar(Q_FULL + sq));
        if (n >= kOSlots) ok = s2_wait(bar(O_EMPTY + so), ((n / kOSlots) - 1) & 1, abort_flag, status, 8);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(O_FULL + so), L::kTileBytes + L::kRowBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(sdO(so) + c * kChunkBytes, &tmdO, c * 64, u.h, row_base + q0, bar(O_FULL + so));
        bulk_load(sb + L::kDelta + so * L::kRowBytes, delta + stat_base + q0, L::kRowBytes, bar(O_FULL + so));
        ++n;
      }
      // the last loads must land before the CTA retires (also after an abort)
      s2_wait_drain(bar(KV_FULL), 0, status, 8);
      for (int d = (n > kQSlots ? n - kQSlots : 0); d < n; ++d)
        s2_wait_drain(bar(Q_FULL + d % kQSlots), (d / kQSlots) & 1, status, 8);
      for (int d = (n > kOSlots ? n - kOSlots : 0); d < n; ++d)
        s2_wait_drain(bar(O_FULL + d % kOSlots), (d / kOSlots) & 1, status, 8);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && kvalid) {
      constexpr uint32_t id_s = umma_idesc_bf16(128, 128, 0, 0);  // S^T, dP^T: M keys, N queries, K-major
      constexpr uint32_t id_acc = umma_idesc_bf16(128, D, 0, 1);  // dV, dK: A from TMEM, B MN-major
      // Descriptors are built once; each MMA adds a compile-time offset.
      const uint64_t dK_km = umma_desc_sw128(sK, 16, 1024), dV_km = umma_desc_sw128(sV, 16, 1024);
      const uint64_t dQ_km = umma_desc_sw128(sQ(0), 16, 1024), ddO_km = umma_desc_sw128(sdO(0), 16, 1024);
      const uint64_t dQ_mn = umma_desc_sw128(sQ(0), kChunkBytes, 1024);
      const uint64_t ddO_mn = umma_desc_sw128(sdO(0), kChunkBytes, 1024);
      constexpr uint64_t kSlotStep = (uint64_t)(L::kTileBytes >> 4);
      bool ok = s2_wait(bar(KV_FULL), 0, abort_flag, status, 16);
      if (ok) ok = s2_wait(bar(Q_FULL + 0), 0, abort_flag, status, 16);
      tc_fence_after();
      if (ok) {  // S(0)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) umma_ss(tR1, dK_km + S2_KM_OFF(kk), dQ_km + S2_KM_OFF(kk), id_s, kk > 0);
        umma_commit(bar(S_FULL));
      }
      int n = 0;
      if (ok) ok = s2_wait(bar(O_FULL + 0), 0, abort_flag, status, 16);
      int qn = next_q(p, u, q_first, lK, hK);
      for (int qt = q_first; ok && qt >= 0;) {
        const int sq = n % kQSlots, sd = n % kOSlots;
        const uint64_t oq = (uint64_t)sq * kSlotStep, od = (uint64_t)sd * kSlotStep;
        // dP^T(n) -> R2 (dO(n) has landed)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tR2, dV_km + S2_KM_OFF(kk), ddO_km + od + S2_KM_OFF(kk), id_s, kk > 0);
        umma_commit(bar(DP_FULL));
        // dV += P^T(n) dO(n): K = 128 queries, 16 per step, P^T pairs at R1 + 64·(kk/4) + 8·(kk%4)
        ok = s2_wait(bar(P_READY), n & 1, abort_flag, status, 16);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tdV, tR1 + 64 * (kk / 4) + 8 * (kk % 4), ddO_mn + od + S2_MN_OFF(kk), id_acc,
                  (n > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(O_EMPTY + sd));  // dV is the last MMA reading dO(n)
        // S^T(n+1) -> R1
        if (qn >= 0) {
          const int sq1 = (n + 1) % kQSlots;
          ok = s2_wait(bar(Q_FULL + sq1), ((n + 1) / kQSlots) & 1, abort_flag, status, 16);
          if (!ok) break;
          const uint64_t oq1 = (uint64_t)sq1 * kSlotStep;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tR1, dK_km + S2_KM_OFF(kk), dQ_km + oq1 + S2_KM_OFF(kk), id_s, kk > 0);
          umma_commit(bar(S_FULL));
        }
        // the next tile and its dO, while S(n+1) is queued
        const int qnn = qn >= 0 ? next_q(p, u, qn, lK, hK) : -1;
        if (qn >= 0) {
          const int sd1 = (n + 1) % kOSlots;
          ok = s2_wait(bar(O_FULL + sd1), ((n + 1) / kOSlots) & 1, abort_flag, status, 16);
          if (!ok) break;
        }
        // dK += dS^T(n) Q(n), dS^T pairs at R2 + 64·(kk/4) + 8·(kk%4)
        ok = s2_wait(bar(DS_READY), n & 1, abort_flag, status, 16);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tdK, tR2 + 64 * (kk / 4) + 8 * (kk % 4), dQ_mn + oq + S2_MN_OFF(kk), id_acc,
                  (n > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(Q_EMPTY + sq));
        ++n;
        qt = qn;
        qn = qnn;
      }
      // every issued MMA must be complete before TMEM is read or released (also after an abort)
      umma_commit(bar(ACC_DONE));
      s2_wait_drain(bar(ACC_DONE), 0, status, 16);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise warpgroups
    const int x = warp / 4;                // query columns [64x, 64x + 64)
    const int j = (warp % 4) * 32 + lane;  // key row == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    bool ok = true;
    int n = 0;
    // R1, R2, dV, dK within the 512 allocated columns
    if (!S2_IN(kSiteKvTmem, 256 + 2 * D, 257, 513)) *abort_flag = 1;
    if (kvalid) {
      const bool key_tile_ragged = k0 + kTile > p.n_valid;
      const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
      // P of the current tile as bf16 pairs, from its exponentials to its dS: dS uses
      // the same rounded P as dV += P^T dO
      uint32_t pk[32];
      // P(nn): S^T -> P^T (bf16 pairs into R1 and pk); the row's 64 columns in one load
      auto p_step = [&](int nn, int qtile) -> bool {
        const int sq = nn % kQSlots;
        // masks on the diagonal tile, on a key tile with padding and under a
        // document mask; padded queries are zeroed by their -inf statistic
        const bool masked = (qtile == kt) || key_tile_ragged || p.docs != nullptr;
        int lo = 0, hi = kTile;
        if (masked) key_cols(p, u, kt, qtile, j, lo, hi);
        if (!s2_wait(bar(Q_FULL + sq), (nn / kQSlots) & 1, abort_flag, status, 32)) return false;
        if (!s2_wait(bar(S_FULL), nn & 1, abort_flag, status, 32)) return false;
        tc_fence_after();
        const float2* nl = reinterpret_cast<const float2*>(smem + L::kLse + sq * L::kRowBytes) + 32 * x;
        uint32_t sv[64];
        tmem_ld64(tR1 + lane_off + 64 * x, sv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          // P = 2^(S·log2(e)/sqrt(D) - lse·log2(e)), two columns at a time
          const float2 a = __ffma2_rn(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), c2, nl[i]);
          float p0 = ex2(a.x), p1 = ex2(a.y);
          if (masked) {
            const int col = 64 * x + 2 * i;
            p0 = (col >= lo && col < hi) ? p0 : 0.f;
            p1 = (col + 1 >= lo && col + 1 < hi) ? p1 : 0.f;
          }
          pk[i] = pack_bf16(p0, p1);
        }
        // P^T pairs over the S columns [64x, 64x + 32), all read already
        tmem_st32(tR1 + lane_off + 64 * x, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(P_READY));
        return true;
      };
      int qt = q_first;
      ok = p_step(0, qt);
      while (ok && qt >= 0) {
        const int sd = n % kOSlots;
        const int qn = next_q(p, u, qt, lK, hK);
        // stored dS of tile (qt, kt): the 16-byte block of key row j and query columns
        // [8b, 8b + 8) sits at (j / 8)·2048 + b·128 + (j % 8)·16 bytes, so one block
        // of a warp's 32 rows is four 128-byte runs
        uint4* ds_tile = nullptr;
        if constexpr (kStoreDS) {
          const long long slot = ds_slot(p, u, qt, kt);
          if (!S2_IN(kSiteKvDs, slot, 0, (long long)p.B * p.H * p.ds_head_tiles)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          ds_tile = reinterpret_cast<uint4*>(ds_store + slot * (kTile * kTile)) + (j >> 3) * 128 + (j & 7);
        }
        // dS(n) = P (dP - Delta) -> dS^T pairs into R2
        ok = s2_wait(bar(O_FULL + sd), (n / kOSlots) & 1, abort_flag, status, 32);
        if (ok) ok = s2_wait(bar(DP_FULL), n & 1, abort_flag, status, 32);
        if (!ok) break;
        tc_fence_after();
        const float2* nd = reinterpret_cast<const float2*>(smem + L::kDelta + sd * L::kRowBytes) + 32 * x;
        uint32_t dp[64];
        tmem_ld64(tR2 + lane_off + 64 * x, dp);
        tmem_wait_ld();
        uint32_t keep[32];  // this row's dS pairs (also stored after the hand-off)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 d2 = __fadd2_rn(make_float2(__uint_as_float(dp[2 * i]), __uint_as_float(dp[2 * i + 1])), nd[i]);
          const float2 pv = make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xffff0000u));
          const float2 ds = __fmul2_rn(pv, d2);
          keep[i] = pack_bf16(ds.x, ds.y);
        }
        tmem_st32(tR2 + lane_off + 64 * x, keep);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(DS_READY));
        mbar_arrive(bar(O_EMPTY + sd));  // done with the -Delta rows of dO slot sd
        if constexpr (kStoreDS) {
          // after the hand-off, so that draining the stores never holds up dK += dS^T Q;
          // evict-first: the dQ pass reads these tiles after the whole pass
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            __stcs(ds_tile + (8 * x + v4) * 8, make_uint4(keep[4 * v4], keep[4 * v4 + 1], keep[4 * v4 + 2], keep[4 * v4 + 3]));
        }
        if (qn >= 0) {
          ok = p_step(n + 1, qn);
          if (!ok) break;
        }
        ++n;
        qt = qn;
      }
    }
    // ---------------------------------------------------------- epilogue: dK, dV
    bool have = kvalid && ok && n > 0;
    if (have) {
      have = s2_wait(bar(ACC_DONE), 0, abort_flag, status, 32);
      tc_fence_after();
    }
    const bool key_valid = k0 + j < p.n_valid;
    const float scale = p.scale_log2 * 0.69314718055994531f;  // 1/sqrt(D)
    // staging: dV -> Q slot 0, dK -> Q slot 1 (every MMA reading them has completed)
    acc_to_smem<D>(tdV, lane_off, x, j, have, key_valid, 1.f, sQ(0));
    acc_to_smem<D>(tdK, lane_off, x, j, have, key_valid, scale, sQ(1));
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 0 && S2_IN(kSiteKvOut, k0, 0, p.N - kTile + 1) &&
        S2_IN(kSiteKvOut, row_base + k0, 0, (long long)p.B * p.N - kTile + 1)) {
      for (int c = 0; c < kChunks; ++c) {
        tma_store_3d(&tmdV, sQ(0) + c * kChunkBytes, c * 64, u.h, row_base + k0);
        tma_store_3d(&tmdK, sQ(1) + c * kChunkBytes, c * 64, u.h, row_base + k0);
      }
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
#undef bar
#undef sQ
#undef sdO
}

// ------------------------------------------------------------------ dQ pass
// Tensor memory (512 columns): S0, S1 [0, 256) double-buffered scores (then
// dS as bf16 pairs in the first half of each warpgroup's 64 columns);
// dP [256, 384); dQ [384, 384 + D).  Key tiles j of the unit, in order; the
// issue order (one thread of warp 9) is
//   S(0), S(1), dP(0), then per j:  dQ += dS(j) K(j),  dP(j+1),  S(j+2)
// so the exponentials of tile j+1 overlap dQ(j) and dP(j+1).  K tiles live in
// a ring of three slots (K(j) is read by S(j) and, two tiles later, dQ(j)),
// V tiles in a ring of two.  Elementwise thread = query row (TMEM lane),
// warpgroup x = key columns [64x, 64x + 64).
namespace dqp {

constexpr int kKSlots = 3, kVSlots = 2;
enum Bar {
  Q_FULL = 0,
  K_FULL = 1,    // + slot (3)
  K_EMPTY = 4,   // + slot (3)
  V_FULL = 7,    // + slot (2)
  V_EMPTY = 9,   // + slot (2)
  S_FULL = 11,   // + buffer (2)
  DP_FULL = 13,
  DS_READY = 14,
  DQ_DONE = 15,
  NUM_BARS = 16
};

template <int D>
struct Layout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kdO = kTileBytes;
  static constexpr int kK = 2 * kTileBytes;                // + slot * kTileBytes
  static constexpr int kV = kK + kKSlots * kTileBytes;      // + slot * kTileBytes
  static constexpr int kBars = kV + kVSlots * kTileBytes;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
};

}  // namespace dqp

template <int D>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    s2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ Plan p,
                     const float* __restrict__ delta,
                     const float* __restrict__ lse2, int* __restrict__ status) {
  using namespace bwd;
  using namespace dqp;
  using L = dqp::Layout<D>;
  constexpr int kChunks = D / 64;

  Unit u;
  if (!decode_q_unit(p, blockIdx.x, u)) return;
  extern __shared__ __align__(1024) uint8_t smem_dq[];
  if (smem_u32(smem_dq) & 1023u) {
    if (threadIdx.x == 0) atomicOr(status, 256);
    return;
  }
  const int qt = u.t[0];
  const int q0 = tile_orig(p, u, qt);
  const bool qvalid = u.part[0];  // the query tile holds a valid row
  int lQ = 0, hQ = p.N;           // span of the documents touching the query tile
  if (qvalid) doc_span(p, u.b, q0, lQ, hQ);

  uint8_t* smem = smem_dq;
  const uint32_t sb = smem_u32(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbar = sb + L::kBars;
#define bar(i) (sbar + 8u * (uint32_t)(i))
#define sKs(slot) (sb + L::kK + (uint32_t)(slot) * L::kTileBytes)
#define sVs(slot) (sb + L::kV + (uint32_t)(slot) * L::kTileBytes)
  const uint32_t sQ = sb + L::kQ, sdO = sb + L::kdO;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar(Q_FULL), 1);
    for (int i = 0; i < kKSlots; ++i) {
      mbar_init(bar(K_FULL + i), 1);
      mbar_init(bar(K_EMPTY + i), 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(bar(V_FULL + i), 1);
      mbar_init(bar(V_EMPTY + i), 1);
    }
    mbar_init(bar(S_FULL + 0), 1);
    mbar_init(bar(S_FULL + 1), 1);
    mbar_init(bar(DP_FULL), 1);
    mbar_init(bar(DS_READY), 256);
    mbar_init(bar(DQ_DONE), 1);
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
  const uint32_t tDP = tmem + 256, tdQ = tmem + 384;
  const int row_base = u.b * p.N;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && qvalid) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(bar(Q_FULL), 2 * L::kTileBytes);
      if (S2_IN(kSiteDqQ, q0, p.q_begin, p.n_valid) && S2_IN(kSiteDqQ, q0, 0, p.N - kTile + 1) &&
          S2_IN(kSiteDqQ, row_base + q0, 0, (long long)p.B * p.N - kTile + 1)) {
        for (int c = 0; c < kChunks; ++c) {
          tma_load_3d(sQ + c * kChunkBytes, &tmQ, c * 64, u.h, row_base + q0, bar(Q_FULL));
          tma_load_3d(sdO + c * kChunkBytes, &tmdO, c * 64, u.h, row_base + q0, bar(Q_FULL));
        }
      } else {
        *abort_flag = 1;
      }
      int eK = 0, eV = 0;
      bool ok = true;
      auto load = [&](bool isK, int k) {
        if (!ok) return;
        const int e = isK ? eK : eV, slots = isK ? kKSlots : kVSlots;
        const int slot = e % slots;
        const uint32_t full = bar((isK ? K_FULL : V_FULL) + slot), empty = bar((isK ? K_EMPTY : V_EMPTY) + slot);
        if (e >= slots) ok = s2_wait(empty, ((e / slots) - 1) & 1, abort_flag, status, 1);
        if (!ok) return;
        mbar_arrive_expect_tx(full, L::kTileBytes);
        const uint32_t dst = isK ? sKs(slot) : sVs(slot);
        const int x0 = tile_orig(p, u, k);
        const int row = row_base + x0;
        if (S2_IN(kSiteDqK, x0, p.k_begin, p.n_valid) && S2_IN(kSiteDqK, x0, 0, p.N - kTile + 1) &&
            S2_IN(kSiteDqK, row, 0, (long long)p.B * p.N - kTile + 1)) {
          for (int c = 0; c < kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, isK ? &tmK : &tmV, c * 64, u.h, row, full);
        } else {
          *abort_flag = 1;
        }
        if (isK) ++eK; else ++eV;
      };
      // consumption order: K(0), K(1), V(0), then per j: V(j+1), K(j+2)
      int ka = next_k(p, u, -1, lQ, hQ);
      int kb = ka >= 0 ? next_k(p, u, ka, lQ, hQ) : -1;
      int kc = kb >= 0 ? next_k(p, u, kb, lQ, hQ) : -1;
      if (ka >= 0) load(true, ka);
      if (kb >= 0) load(true, kb);
      if (ka >= 0) load(false, ka);
      while (ok && ka >= 0) {
        if (kb >= 0) load(false, kb);
        if (kc >= 0) load(true, kc);
        ka = kb;
        kb = kc;
        kc = kc >= 0 ? next_k(p, u, kc, lQ, hQ) : -1;
      }
      // the last loads must land before the CTA retires (also after an abort)
      for (int d = (eK > kKSlots ? eK - kKSlots : 0); d < eK; ++d)
        s2_wait_drain(bar(K_FULL + d % kKSlots), (d / kKSlots) & 1, status, 1);
      for (int d = (eV > kVSlots ? eV - kVSlots : 0); d < eV; ++d)
        s2_wait_drain(bar(V_FULL + d % kVSlots), (d / kVSlots) & 1, status, 1);
      s2_wait_drain(bar(Q_FULL), 0, status, 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && qvalid) {
      constexpr uint32_t id_s = umma_idesc_bf16(128, 128, 0, 0);  // S, dP: M queries, N keys, K-major
      constexpr uint32_t id_q = umma_idesc_bf16(128, D, 0, 1);    // dQ: A = dS from TMEM, B = K MN-major
      const uint64_t dQ_km = umma_desc_sw128(sQ, 16, 1024), ddO_km = umma_desc_sw128(sdO, 16, 1024);
      const uint64_t dK_km = umma_desc_sw128(sKs(0), 16, 1024), dV_km = umma_desc_sw128(sVs(0), 16, 1024);
      const uint64_t dK_mn = umma_desc_sw128(sKs(0), kChunkBytes, 1024);
      constexpr uint64_t kSlotStep = (uint64_t)(L::kTileBytes >> 4);
      int T = 0;  // key tiles of this unit
      for (int k = next_k(p, u, -1, lQ, hQ); k >= 0; k = next_k(p, u, k, lQ, hQ)) ++T;
      bool ok = s2_wait(bar(Q_FULL), 0, abort_flag, status, 2);
      auto issue_s = [&](int jj) {  // S(jj) = Q K(jj)^T -> S buffer jj % 2 (K(jj) has landed)
        const int slot = jj % kKSlots;
        if (!ok) return;
        const uint64_t so = (uint64_t)slot * kSlotStep;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + 128 * (jj % 2), dQ_km + S2_KM_OFF(kk), dK_km + so + S2_KM_OFF(kk), id_s, kk > 0);
        umma_commit(bar(S_FULL + (jj % 2)));
      };
      auto issue_dp = [&](int jj) {  // dP(jj) = dO V(jj)^T -> dP (V(jj) has landed)
        const int slot = jj % kVSlots;
        if (!ok) return;
        const uint64_t so = (uint64_t)slot * kSlotStep;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tDP, ddO_km + S2_KM_OFF(kk), dV_km + so + S2_KM_OFF(kk), id_s, kk > 0);
        umma_commit(bar(DP_FULL));
        umma_commit(bar(V_EMPTY + slot));
      };
      auto wait_k = [&](int jj) {
        ok = ok && s2_wait(bar(K_FULL + jj % kKSlots), (jj / kKSlots) & 1, abort_flag, status, 2);
      };
      auto wait_v = [&](int jj) {
        ok = ok && s2_wait(bar(V_FULL + jj % kVSlots), (jj / kVSlots) & 1, abort_flag, status, 2);
      };
      if (T > 0) { wait_k(0); issue_s(0); }
      if (T > 1) { wait_k(1); issue_s(1); }
      if (T > 0) { wait_v(0); issue_dp(0); }
      for (int jj = 0; ok && jj < T; ++jj) {
        // the loads this iteration consumes first (landed long ago, as a rule), then the
        // dS hand-off: the three batches below then issue back to back
        if (jj + 1 < T) wait_v(jj + 1);
        if (jj + 2 < T) wait_k(jj + 2);
        if (ok) ok = s2_wait(bar(DS_READY), jj & 1, abort_flag, status, 2);
        if (!ok) break;
        tc_fence_after();
        // dQ += dS(jj) K(jj): K = 128 keys, 16 per step, dS pairs at S + 64·(kk/4) + 8·(kk%4)
        const int slot = jj % kKSlots;
        const uint64_t so = (uint64_t)slot * kSlotStep;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tdQ, tmem + 128 * (jj % 2) + 64 * (kk / 4) + 8 * (kk % 4), dK_mn + so + S2_MN_OFF(kk), id_q,
                  (jj > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(K_EMPTY + slot));
        if (jj + 1 < T) issue_dp(jj + 1);  // dP(jj) was read before DS_READY(jj)
        if (jj + 2 < T) issue_s(jj + 2);   // behind dQ(jj), the last reader of this S buffer
      }
      // every issued MMA must be complete before TMEM is read or released (also after an abort)
      umma_commit(bar(DQ_DONE));
      s2_wait_drain(bar(DQ_DONE), 0, status, 2);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise warpgroups
    const int x = warp / 4;                // key columns [64x, 64x + 64)
    const int r = (warp % 4) * 32 + lane;  // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const bool row_valid = q0 + r < p.n_valid;
    bool ok = true;
    int jj = 0;
    if (qvalid) {
      const size_t stat_at = ((size_t)u.b * p.H + u.h) * p.N + q0 + r;
      // S0, S1, dP, dQ within the 512 allocated columns; the row's statistics
      if (!(S2_IN(kSiteDqTmem, 384 + D, 385, 513) && S2_IN(kSiteDqQ, stat_at, 0, (long long)p.B * p.H * p.N)))
        *abort_flag = 1;
      const float nl = lse2[stat_at], nd = delta[stat_at];  // -lse·log2(e) (-inf if padded), -Delta
      const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
      const float2 nl2 = make_float2(nl, nl), nd2 = make_float2(nd, nd);
      for (int k = next_k(p, u, -1, lQ, hQ); ok && k >= 0; k = next_k(p, u, k, lQ, hQ), ++jj) {
        const uint32_t tS = tmem + 128 * (jj % 2);
        // key columns [cmin, cmax) of this tile are visible from row r (causal diagonal,
        // padding, the row's document)
        int cmin, cmax;
        row_cols(p, u, qt, k, r, cmin, cmax);
        const bool masked = !__all_sync(0xffffffffu, cmin == 0 && cmax == kTile);
        ok = s2_wait(bar(S_FULL + (jj % 2)), (jj / 2) & 1, abort_flag, status, 4);
        if (!ok) break;
        tc_fence_after();
        // the row's 64 columns in one load; P kept as the bf16 pairs
        // dS is formed from (the same rounding as the dK/dV pass)
        uint32_t sv[64];
        tmem_ld64(tS + lane_off + 64 * x, sv);
        tmem_wait_ld();
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 a = __ffma2_rn(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), c2, nl2);
          float p0 = ex2(a.x), p1 = ex2(a.y);
          if (masked) {
            const int col = 64 * x + 2 * i;
            p0 = (col >= cmin && col < cmax) ? p0 : 0.f;
            p1 = (col + 1 >= cmin && col + 1 < cmax) ? p1 : 0.f;
          }
          pk[i] = pack_bf16(p0, p1);
        }
        ok = s2_wait(bar(DP_FULL), jj & 1, abort_flag, status, 4);
        if (!ok) break;
        tc_fence_after();
        uint32_t dp[64];
        tmem_ld64(tDP + lane_off + 64 * x, dp);
        tmem_wait_ld();
        uint32_t dsp[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 d2 = __fadd2_rn(make_float2(__uint_as_float(dp[2 * i]), __uint_as_float(dp[2 * i + 1])), nd2);
          const float2 pv = make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xffff0000u));
          const float2 ds = __fmul2_rn(pv, d2);
          dsp[i] = pack_bf16(ds.x, ds.y);
        }
        // dS pairs of key columns [64x, 64x + 64) -> S columns 64x + [0, 32), already read
        tmem_st32(tS + lane_off + 64 * x, dsp);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(DS_READY));
      }
    }
    // ---------------------------------------------------------- epilogue: dq
    bool have = qvalid && ok && jj > 0;
    if (have) {
      have = s2_wait(bar(DQ_DONE), 0, abort_flag, status, 4);
      tc_fence_after();
    }
    const float scale = p.scale_log2 * 0.69314718055994531f;  // 1/sqrt(D)
    // staging in the Q tile (every MMA reading it has completed)
    acc_to_smem<D>(tdQ, lane_off, x, r, have, row_valid, scale, sQ);
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 0 && S2_IN(kSiteDqOut, q0, 0, p.N - kTile + 1) &&
        S2_IN(kSiteDqOut, row_base + q0, 0, (long long)p.B * p.N - kTile + 1)) {
      for (int c = 0; c < kChunks; ++c) tma_store_3d(&tmdQ, sQ + c * kChunkBytes, c * 64, u.h, row_base + q0);
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
#undef bar
#undef sKs
#undef sVs
}

// ------------------------------------------------------------------ dQ from stored dS
// One CTA per 128-query tile: dQ = sum over the unit's key tiles of dS K,
// with dS read back from the dK/dV pass and K as an MN-major B operand.  A
// stored tile (32 KB, contiguous) is already the unswizzled canonical layout
// of an MN-major operand: core matrices of 8 key rows x 8 query columns (128
// contiguous bytes), 128 bytes apart along M (queries) and 2048 bytes apart
// along K (keys), so the 16 core matrices one K group reads are 2 KB of
// consecutive banks.  One bulk copy moves a tile.  No exponentials, no recomputed products: the pass
// streams 32 KB of dS per key tile from HBM and is bounded by that.  Warp 8
// loads (dS tile + K tile per stage, three stages), one thread of warp 9
// issues the MMAs, warps 0-7 run the epilogue (dq = bf16(dQ/sqrt(D)) through
// a TMA store).
namespace dqs {

constexpr int kStages = 3;
enum Bar { FULL = 0, EMPTY = 3, DQ_DONE = 6, NUM_BARS = 7 };

template <int D>
struct Layout {
  static constexpr int kDSBytes = kTile * kTile * 2;
  static constexpr int kKBytes = kTile * D * 2;
  static constexpr int kStageBytes = kDSBytes + kKBytes;
  static constexpr int kBars = kStages * kStageBytes;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
};

}  // namespace dqs

template <int D>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    s2_bwd_dq_ds_kernel(const __grid_constant__ CUtensorMap tmK, const __nv_bfloat16* __restrict__ ds,
                        const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ Plan p,
                        int* __restrict__ status) {
  using namespace bwd;
  using namespace dqs;
  using L = dqs::Layout<D>;
  constexpr int kChunks = D / 64;

  Unit u;
  if (!decode_q_unit(p, blockIdx.x, u)) return;
  extern __shared__ __align__(1024) uint8_t smem_dqs[];
  if (smem_u32(smem_dqs) & 1023u) {
    if (threadIdx.x == 0) atomicOr(status, 256);
    return;
  }
  const int qt = u.t[0];
  const int q0 = tile_orig(p, u, qt);
  const bool qvalid = u.part[0];
  int lQ = 0, hQ = p.N;
  if (qvalid) doc_span(p, u.b, q0, lQ, hQ);

  uint8_t* smem = smem_dqs;
  const uint32_t sb = smem_u32(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbar = sb + L::kBars;
#define bar(i) (sbar + 8u * (uint32_t)(i))
#define sDS(st) (sb + (uint32_t)(st) * L::kStageBytes)
#define sKt(st) (sb + (uint32_t)(st) * L::kStageBytes + L::kDSBytes)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(FULL + i), 1);
      mbar_init(bar(EMPTY + i), 1);
    }
    mbar_init(bar(DQ_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), D);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tdQ = *tmem_slot;
  const int row_base = u.b * p.N;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && qvalid) {
      prefetch_tmap(&tmK);
      int e = 0;
      bool ok = true;
      for (int k = next_k(p, u, -1, lQ, hQ); ok && k >= 0; k = next_k(p, u, k, lQ, hQ), ++e) {
        const int st = e % kStages;
        if (e >= kStages) ok = s2_wait(bar(EMPTY + st), ((e / kStages) - 1) & 1, abort_flag, status, 1);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(FULL + st), L::kStageBytes);
        const long long slot = ds_slot(p, u, qt, k);
        const int x0 = tile_orig(p, u, k);
        const int row = row_base + x0;
        if (S2_IN(kSiteDqK, slot, 0, (long long)p.B * p.H * p.ds_head_tiles) &&
            S2_IN(kSiteDqK, x0, p.k_begin, p.n_valid) && S2_IN(kSiteDqK, x0, 0, p.N - kTile + 1) &&
            S2_IN(kSiteDqK, row, 0, (long long)p.B * p.N - kTile + 1)) {
          bulk_load(sDS(st), ds + slot * (kTile * kTile), L::kDSBytes, bar(FULL + st));
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(sKt(st) + c * kChunkBytes, &tmK, c * 64, u.h, row, bar(FULL + st));
        } else {
          *abort_flag = 1;
        }
      }
      // the last loads must land before the CTA retires (also after an abort)
      for (int d = (e > kStages ? e - kStages : 0); d < e; ++d)
        s2_wait_drain(bar(FULL + d % kStages), (d / kStages) & 1, status, 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && qvalid) {
      // dQ: M = 128 queries, N = D, K = 128 keys; A = dS (MN-major: queries contiguous), B = K (MN-major)
      constexpr uint32_t id_q = umma_idesc_bf16(128, D, 1, 1);
      const uint64_t dDS_mn = umma_desc_noswz(sDS(0), 2048, 128);  // K: 2048 B, M: 128 B
      const uint64_t dK_mn = umma_desc_sw128(sKt(0), kChunkBytes, 1024);
      constexpr uint64_t kStageStep = (uint64_t)(L::kStageBytes >> 4);
      bool ok = true;
      int jj = 0;
      for (int k = next_k(p, u, -1, lQ, hQ); ok && k >= 0; k = next_k(p, u, k, lQ, hQ), ++jj) {
        const int st = jj % kStages;
        ok = s2_wait(bar(FULL + st), (jj / kStages) & 1, abort_flag, status, 2);
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          // K step kk: 16 keys = two K groups of dS (4096 bytes), 16 rows of K
          umma_ss(tdQ, dDS_mn + so + (uint64_t)(kk * 256), dK_mn + so + S2_MN_OFF(kk), id_q,
                  (jj > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(EMPTY + st));
      }
      // every issued MMA must be complete before TMEM is read or released (also after an abort)
      umma_commit(bar(DQ_DONE));
      s2_wait_drain(bar(DQ_DONE), 0, status, 2);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue: dq
    const int x = warp / 4;
    const int r = (warp % 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const bool row_valid = q0 + r < p.n_valid;
    bool have = qvalid;
    if (have) {
      have = s2_wait(bar(DQ_DONE), 0, abort_flag, status, 4);
      tc_fence_after();
    }
    const float scale = p.scale_log2 * 0.69314718055994531f;  // 1/sqrt(D)
    // staging in stage 0's dS area (every load has landed and every MMA has completed)
    acc_to_smem<D>(tdQ, lane_off, x, r, have, row_valid, scale, sDS(0));
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 0 && S2_IN(kSiteDqOut, q0, 0, p.N - kTile + 1) &&
        S2_IN(kSiteDqOut, row_base + q0, 0, (long long)p.B * p.N - kTile + 1)) {
      for (int c = 0; c < kChunks; ++c) tma_store_3d(&tmdQ, sDS(0) + c * kChunkBytes, c * 64, u.h, row_base + q0);
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tdQ, D);
  }
#undef bar
#undef sDS
#undef sKt
}

#undef S2_KM_OFF
#undef S2_MN_OFF

template <int D, bool kStoreDS>
int launch_dkdv(const BwdArgs& a, int grid) {
  constexpr int kBytes = dkdv::Layout<D>::kBytes;
  cudaError_t e =
      cudaFuncSetAttribute(s2_bwd_dkdv_kernel<D, kStoreDS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBytes);
  if (e != cudaSuccess) return (int)e;
  s2_bwd_dkdv_kernel<D, kStoreDS><<<grid, bwd::kThreads, kBytes, a.stream>>>(
      *a.tmQ, *a.tmK, *a.tmV, *a.tmdO, *a.tmdK, *a.tmdV, a.plan, a.delta, a.lse2,
      static_cast<__nv_bfloat16*>(a.ds), a.status);
  return (int)cudaGetLastError();
}

template <int D>
int launch_bwd_impl(const BwdArgs& a, int stages) {
  static_assert(dkdv::Layout<D>::kBytes <= 232448 && dqp::Layout<D>::kBytes <= 232448 &&
                    dqs::Layout<D>::kBytes <= 232448,
                "shared memory budget");
  const bool stored = (stages & 8) != 0;
  const Plan& p = a.plan;
  const long long rows = (long long)p.B * p.N * p.H;
  cudaError_t e;
  if (stages & 1) {  // prepare: -Delta and -lse·log2(e)
    constexpr int kRowsPerBlock = 256 / (D / 8);
    s2_bwd_pre<D><<<(unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.lse, a.delta, a.lse2,
        p.B, p.N, p.H, p.q_begin, p.n_valid);
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
  }
  const int grid = grid_bwd(p);
  if (stages & 2) {  // dK, dV (and the stored dS)
    const int rc = stored ? launch_dkdv<D, true>(a, grid) : launch_dkdv<D, false>(a, grid);
    if (rc) return rc;
  }
  if ((stages & 4) && stored) {  // dQ from the stored dS
    constexpr int kBytes = dqs::Layout<D>::kBytes;
    e = cudaFuncSetAttribute(s2_bwd_dq_ds_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBytes);
    if (e != cudaSuccess) return (int)e;
    s2_bwd_dq_ds_kernel<D><<<grid, bwd::kThreads, kBytes, a.stream>>>(
        *a.tmK, static_cast<const __nv_bfloat16*>(a.ds), *a.tmdQ, p, a.status);
  } else if (stages & 4) {  // dQ
    constexpr int kBytes = dqp::Layout<D>::kBytes;
    e = cudaFuncSetAttribute(s2_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBytes);
    if (e != cudaSuccess) return (int)e;
    s2_bwd_dq_kernel<D><<<grid, bwd::kThreads, kBytes, a.stream>>>(*a.tmQ, *a.tmK, *a.tmV, *a.tmdO, *a.tmdQ, p,
                                                                  a.delta, a.lse2, a.status);
  }
  return (int)cudaGetLastError();
}

int launch_bwd(const BwdArgs& a, int stages) {
  if (a.plan.D == 64) return launch_bwd_impl<64>(a, stages);
  return launch_bwd_impl<128>(a, stages);
}

}  // namespace s2
