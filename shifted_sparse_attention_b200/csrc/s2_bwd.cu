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
// Three kernels on the caller's stream:
//   1. s2_bwd_pre: -Delta_i = -(dout_i·o_i) and -lse_i·log2(e) (-inf on
//      padded rows, which zeroes their probabilities), per [B, H, N].
//   2. s2_bwd_kernel: one CTA per 128-key tile of a segment, walking the
//      query tiles from the diagonal to the segment's end:
//        S^T  = K Q^T        (TMEM)            dP^T = V dO^T     (TMEM)
//        P^T  = exp2(S^T·c - lse2), dS^T = P^T (dP^T - Delta)   (CUDA cores)
//        dV  += P^T dO       (A from TMEM)     dK  += dS^T Q     (TMEM)
//        dQ_i = dS K         (TMEM) -> added into a float32 accumulator.
//      dK, dV leave through a TMA store at the end.
//   3. s2_bwd_dq_convert: dq = bf16(scale · accumulator).
// Warp roles of s2_bwd_kernel (320 threads): warps 0-7 elementwise work, the
// two warpgroups splitting the 128 query columns in halves (thread = one key
// row = one TMEM lane); warp 8 TMA producer; warp 9 TMEM allocator and MMA
// issuer.  TMEM (512 columns): S^T / P^T [0,128), dP^T / dQ [128,256),
// dV [256, 256+D), dK [256+D, 256+2D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_index.cuh"
#include "s2_kernels.h"
#include "sm100_ptx.cuh"

namespace s2 {

namespace bwd {

constexpr int kThreads = 320;
constexpr int kStages = 2;
constexpr int kChunkBytes = kTile * 64 * 2;

enum Bar {
  KV_FULL = 0,
  QD_FULL = 1,   // + stage (2)
  QD_EMPTY = 3,  // + stage (2)
  S_FULL = 5,
  DP_FULL = 6,
  DS_READY = 7,
  DV_DONE = 8,
  DQ_FULL = 9,
  DQ_FREE = 10,
  ACC_DONE = 11,
  S_READ = 12,   // both elementwise warpgroups have read S^T (before P^T overwrites it)
  NUM_BARS = 13
};

template <int D>
struct Layout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kTileBytes;
  static constexpr int kQ = 2 * kTileBytes;                    // + stage * kTileBytes
  static constexpr int kdO = kQ + kStages * kTileBytes;        // + stage * kTileBytes
  static constexpr int kdS = kdO + kStages * kTileBytes;       // 128 x 128 bf16
  static constexpr int kBars = kdS + kTile * kTile * 2;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ int next_q(const Plan& p, const Unit& u, int qt) {
  for (int j = qt + 1; j <= u.kmax; ++j)
    if (ktile_valid(p, u, j)) return j;
  return -1;
}

}  // namespace bwd

// ------------------------------------------------------------------ preprocess
// kTpr = D/8 threads per (b, i, h) row, 8 bf16 (16 bytes) each.  Stores the
// negated statistics the main kernel adds: -Delta = -(dout·o) and
// -lse·log2(e) (-inf on padded rows, which zeroes their probabilities).
template <int D>
__global__ void __launch_bounds__(256) s2_bwd_pre(const __nv_bfloat16* __restrict__ o,
                                                   const __nv_bfloat16* __restrict__ dout,
                                                   const float* __restrict__ lse, float* __restrict__ delta,
                                                   float* __restrict__ lse2, int B, int N, int H, int n_valid) {
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
    const bool valid = i < n_valid;
    delta[at] = valid ? -acc : 0.f;
    lse2[at] = valid ? -lse[at] * 1.4426950408889634f : -INFINITY;
  }
}

// ------------------------------------------------------------------ dq convert
__global__ void __launch_bounds__(256) s2_bwd_dq_convert(const float4* __restrict__ acc,
                                                          uint2* __restrict__ dq, long long n4, float scale) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 a = acc[i];
    uint2 r;
    r.x = pack_bf16(a.x * scale, a.y * scale);
    r.y = pack_bf16(a.z * scale, a.w * scale);
    dq[i] = r;
  }
}

// ------------------------------------------------------------------ main backward kernel
template <int D>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    s2_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                  const Plan p, const float* __restrict__ delta, const float* __restrict__ lse2,
                  float* __restrict__ dq_acc, int* __restrict__ status) {
  using namespace bwd;
  using L = Layout<D>;
  constexpr int kChunks = D / 64;

  Unit u;
  if (!decode_kv_unit(p, blockIdx.x, u)) return;
  const int kt = u.t[0];
  const int k0 = tile_orig(p, u, kt);
  const bool kvalid = u.part[0];

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const uint32_t sK = sb + L::kK, sV = sb + L::kV, sdS = sb + L::kdS;
  auto sQ = [&](int st) { return sb + L::kQ + st * L::kTileBytes; };
  auto sdO = [&](int st) { return sb + L::kdO + st * L::kTileBytes; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar(KV_FULL), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(QD_FULL + s), 1);
      mbar_init(bar(QD_EMPTY + s), 1);
    }
    mbar_init(bar(S_FULL), 1);
    mbar_init(bar(DP_FULL), 1);
    mbar_init(bar(DS_READY), 256);
    mbar_init(bar(DV_DONE), 1);
    mbar_init(bar(DQ_FULL), 1);
    mbar_init(bar(DQ_FREE), 256);
    mbar_init(bar(ACC_DONE), 1);
    mbar_init(bar(S_READ), 256);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const int row_base = u.b * p.N;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && kvalid) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(KV_FULL), 2 * L::kTileBytes);
      for (int c = 0; c < kChunks; ++c) {
        tma_load_3d(sK + c * kChunkBytes, &tmK, c * 64, u.h, row_base + k0, bar(KV_FULL));
        tma_load_3d(sV + c * kChunkBytes, &tmV, c * 64, u.h, row_base + k0, bar(KV_FULL));
      }
      int n = 0;
      bool ok = true;
      for (int qt = kt; ok && qt >= 0; qt = next_q(p, u, qt)) {
        if (qt == kt && !ktile_valid(p, u, qt)) continue;
        const int st = n % kStages;
        if (n >= kStages) ok = s2_wait(bar(QD_EMPTY + st), ((n / kStages) - 1) & 1, abort_flag, status, 8);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(QD_FULL + st), 2 * L::kTileBytes);
        const int q0 = tile_orig(p, u, qt);
        for (int c = 0; c < kChunks; ++c) {
          tma_load_3d(sQ(st) + c * kChunkBytes, &tmQ, c * 64, u.h, row_base + q0, bar(QD_FULL + st));
          tma_load_3d(sdO(st) + c * kChunkBytes, &tmdO, c * 64, u.h, row_base + q0, bar(QD_FULL + st));
        }
        ++n;
      }
      for (int d = (n > kStages ? n - kStages : 0); d < n; ++d)
        s2_wait(bar(QD_FULL + d % kStages), (d / kStages) & 1, abort_flag, status, 8);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && kvalid) {
      constexpr uint32_t id_st = umma_idesc_bf16(128, 128, 0, 0);  // S^T, dP^T: K-major A and B
      constexpr uint32_t id_dv = umma_idesc_bf16(128, D, 0, 1);    // dV: A in TMEM, B = dO MN-major
      constexpr uint32_t id_dk = umma_idesc_bf16(128, D, 0, 1);    // dK: A = dS^T K-major, B = Q MN-major
      constexpr uint32_t id_dq = umma_idesc_bf16(128, D, 1, 1);    // dQ: A = dS MN-major, B = K MN-major
      bool ok = s2_wait(bar(KV_FULL), 0, abort_flag, status, 16);
      tc_fence_after();
      int n = 0;
      for (int qt = kt; ok && qt >= 0; qt = next_q(p, u, qt)) {
        if (qt == kt && !ktile_valid(p, u, qt)) continue;
        const int st = n % kStages;
        ok = s2_wait(bar(QD_FULL + st), (n / kStages) & 1, abort_flag, status, 16);
        if (!ok) break;
        tc_fence_after();
        if (n > 0) {  // P^T(n-1) in the S columns must have been consumed by dV(n-1)
          ok = s2_wait(bar(DV_DONE), (n - 1) & 1, abort_flag, status, 16);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kChunkBytes + (kk % 4) * 32;
          umma_ss(tS, umma_desc_sw128(sK + off, 16, 1024), umma_desc_sw128(sQ(st) + off, 16, 1024), id_st, kk > 0);
        }
        umma_commit(bar(S_FULL));
        if (n > 0) {  // dQ(n-1) in the dP columns must have been read out
          ok = s2_wait(bar(DQ_FREE), (n - 1) & 1, abort_flag, status, 16);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kChunkBytes + (kk % 4) * 32;
          umma_ss(tDP, umma_desc_sw128(sV + off, 16, 1024), umma_desc_sw128(sdO(st) + off, 16, 1024), id_st, kk > 0);
        }
        umma_commit(bar(DP_FULL));
        ok = s2_wait(bar(DS_READY), n & 1, abort_flag, status, 16);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO : K = 128 queries, A = P^T packed two per TMEM column
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tdV, tS + kk * 8, umma_desc_sw128(sdO(st) + kk * 2048, kChunkBytes, 1024), id_dv,
                  (n > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(DV_DONE));
        // dK += dS^T Q
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint32_t aoff = (kk / 4) * kChunkBytes + (kk % 4) * 32;
          umma_ss(tdK, umma_desc_sw128(sdS + aoff, 16, 1024),
                  umma_desc_sw128(sQ(st) + kk * 2048, kChunkBytes, 1024), id_dk, (n > 0 || kk > 0) ? 1u : 0u);
        }
        // dQ = dS K : M = 128 queries, K = 128 keys; both operands MN-major
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ss(tDP, umma_desc_sw128(sdS + kk * 2048, kChunkBytes, 1024),
                  umma_desc_sw128(sK + kk * 2048, kChunkBytes, 1024), id_dq, kk > 0 ? 1u : 0u);
        umma_commit(bar(DQ_FULL));
        umma_commit(bar(QD_EMPTY + st));
        ++n;
      }
      umma_commit(bar(ACC_DONE));
      s2_wait(bar(ACC_DONE), 0, abort_flag, status, 16);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise warpgroups
    const int x = warp / 4;            // column half: queries [64x, 64x + 64)
    const int j = (warp % 4) * 32 + lane;  // key row == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const size_t stat_base = ((size_t)u.b * p.H + u.h) * p.N;
    bool ok = true;
    int n = 0;
    if (kvalid) {
      for (int qt = kt; ok && qt >= 0; qt = next_q(p, u, qt)) {
        if (qt == kt && !ktile_valid(p, u, qt)) continue;
        const int q0 = tile_orig(p, u, qt);
        int lo, hi;
        query_range(p, u, kt, qt, j, lo, hi);
        ok = s2_wait(bar(S_FULL), n & 1, abort_flag, status, 32);
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32(tS + lane_off + 64 * x, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tS + lane_off + 64 * x + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        // both halves must have read S^T before either overwrites it with P^T
        mbar_arrive(bar(S_READ));
        ok = s2_wait(bar(S_READ), n & 1, abort_flag, status, 32);
        if (!ok) break;
        ok = s2_wait(bar(DP_FULL), n & 1, abort_flag, status, 32);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col0 = 64 * x + 32 * c;
          uint32_t dp[32];
          tmem_ld32(tDP + lane_off + col0, dp);
          tmem_wait_ld();
          const float4* l4 = reinterpret_cast<const float4*>(lse2 + stat_base + q0 + col0);
          const float4* d4 = reinterpret_cast<const float4*>(delta + stat_base + q0 + col0);
          uint32_t pp[16], dsp[16];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 lv = __ldg(l4 + g), dv = __ldg(d4 + g);
            const float lsv[4] = {lv.x, lv.y, lv.z, lv.w};
            const float dlv[4] = {dv.x, dv.y, dv.z, dv.w};
            float pv[4], dsv[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int i = 4 * g + t;
              const int col = col0 + i;
              const bool vis = (col >= lo) && (col < hi);
              const float pr = vis ? ex2(fmaf(__uint_as_float(sv[32 * c + i]), p.scale_log2, lsv[t])) : 0.f;
              pv[t] = pr;
              dsv[t] = pr * (__uint_as_float(dp[i]) + dlv[t]);
            }
            pp[2 * g] = pack_bf16(pv[0], pv[1]);
            pp[2 * g + 1] = pack_bf16(pv[2], pv[3]);
            dsp[2 * g] = pack_bf16(dsv[0], dsv[1]);
            dsp[2 * g + 1] = pack_bf16(dsv[2], dsv[3]);
          }
          tmem_st16(tS + lane_off + col0 / 2, pp);
          // dS^T row j, columns col0..col0+31: chunk x, 16-byte pieces 4c..4c+3
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int piece = 4 * c + q;
            const uint32_t addr = sdS + x * kChunkBytes + j * 128 + ((piece ^ (j & 7)) << 4);
            st_shared_v4(addr, dsp[4 * q], dsp[4 * q + 1], dsp[4 * q + 2], dsp[4 * q + 3]);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(DS_READY));
        // dQ tile (thread = query row j of this query tile): add into the accumulator
        ok = s2_wait(bar(DQ_FULL), n & 1, abort_flag, status, 32);
        if (!ok) break;
        tc_fence_after();
        const bool qrow_valid = q0 + j < p.n_valid;
#pragma unroll
        for (int c2 = 0; c2 < D / 64; ++c2) {
          const int d0 = x * (D / 2) + 32 * c2;
          uint32_t dq[32];
          tmem_ld32(tDP + lane_off + d0, dq);
          tmem_wait_ld();
          if (qrow_valid) {
            float* dst = dq_acc + (((size_t)row_base + q0 + j) * p.H + u.h) * D + d0;
#pragma unroll
            for (int g = 0; g < 8; ++g)
              red_add_v4(dst + 4 * g, __uint_as_float(dq[4 * g]), __uint_as_float(dq[4 * g + 1]),
                         __uint_as_float(dq[4 * g + 2]), __uint_as_float(dq[4 * g + 3]));
          }
        }
        tc_fence_before();
        mbar_arrive(bar(DQ_FREE));
        ++n;
      }
    }
    // ---------------------------------------------------------- epilogue: dK, dV
    bool have = kvalid && ok && n > 0;
    if (have) {
      have = s2_wait(bar(ACC_DONE), 0, abort_flag, status, 32);
      tc_fence_after();
    }
    const bool key_valid = have && (k0 + j < p.n_valid);
    const float scale = p.scale_log2 * 0.69314718055994531f;  // 1/sqrt(D)
    // staging: dV -> Q stage 0, dK -> Q stage 1 (free once every MMA has completed)
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint32_t tsrc = which == 0 ? tdV : tdK;
      const float mul = which == 0 ? 1.f : scale;
      const uint32_t stage = sQ(which);
#pragma unroll
      for (int c2 = 0; c2 < D / 64; ++c2) {
        const int d0 = x * (D / 2) + 32 * c2;
        uint32_t v[32];
        if (have) {
          tmem_ld32(tsrc + lane_off + d0, v);
          tmem_wait_ld();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = d0 + 8 * q;
          const int chunk = col / 64, piece = (col % 64) / 8;
          uint32_t w[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float a = key_valid ? __uint_as_float(v[8 * q + 2 * t]) * mul : 0.f;
            const float b = key_valid ? __uint_as_float(v[8 * q + 2 * t + 1]) * mul : 0.f;
            w[t] = pack_bf16(a, b);
          }
          st_shared_v4(stage + chunk * kChunkBytes + j * 128 + ((piece ^ (j & 7)) << 4), w[0], w[1], w[2], w[3]);
        }
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 0) {
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
}

// ------------------------------------------------------------------ split backward kernel (D = 128)
// Same CTA decomposition (one 128-key tile, query tiles from the diagonal to
// the segment end), but every query tile is processed as two 64-query halves,
// half x by warpgroup x, so that one half's elementwise work runs while the
// tensor core works on the other half:
//   S^T_x  = K Q_x^T          (M 128 keys, N 64 queries)   TMEM [64x, 64x+64)
//   dP^T_x = V dO_x^T                                        TMEM [128+64x, ...)
//   P^T_x (bf16, into the dP^T_x columns), dS^T_x (bf16, shared memory)
//   dV += P^T_x dO_x (A from TMEM),  dK += dS^T_x Q_x
//   dQ^T_x = K^T dS^T_x       (M = D = 128, N 64 queries) -> the S^T_x columns
// dQ^T puts d on the TMEM lanes, so each warp's float32 atomic adds into the
// dq accumulator cover 128 contiguous bytes of one query row.
namespace bwds {

constexpr int D = 128;
constexpr int kThreads = 320;
constexpr int kStages = 2;
constexpr int kChunkBytes = kTile * 64 * 2;

enum Bar {
  KV_FULL = 0,
  QD_FULL = 1,    // + stage (2)
  QD_EMPTY = 3,   // + stage (2)
  SP_FULL = 5,    // + half (2)
  DS_READY = 7,   // + half (2)
  DQ_FULL = 9,    // + half (2)
  DQ_FREE = 11,   // + half (2)
  ACC_DONE = 13,
  RED_DONE = 14,  // + stage (2): both halves' dQ reductions have read their staging rows
  NUM_BARS = 16
};

struct Layout {
  static constexpr int kTileBytes = kTile * D * 2;       // 32 KB
  static constexpr int kHalfBytes = kTile * 64 * 2;      // 16 KB: dS^T of one half
  static constexpr int kStatBytes = 2 * kTile * 4;       // lse2[128], delta[128]
  static constexpr int kK = 0;
  static constexpr int kV = kTileBytes;
  static constexpr int kQ = 2 * kTileBytes;
  static constexpr int kdO = kQ + kStages * kTileBytes;
  static constexpr int kdS = kdO + kStages * kTileBytes;
  static constexpr int kStat = kdS + 2 * kHalfBytes;
  static constexpr int kBars = kStat + kStages * kStatBytes;
  static constexpr int kBytes = kBars + NUM_BARS * 8 + 16;
};

}  // namespace bwds

__global__ void __launch_bounds__(bwds::kThreads, 1)
    s2_bwd_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                        const __grid_constant__ CUtensorMap tmdQacc, const Plan p, const float* __restrict__ delta,
                        const float* __restrict__ lse2, int* __restrict__ status) {
  using namespace bwds;
  using L = bwds::Layout;
  constexpr int kChunks = D / 64;

  Unit u;
  if (!decode_kv_unit(p, blockIdx.x, u)) return;
  extern __shared__ __align__(1024) uint8_t smem_split[];
  // The layout needs a 1024-byte aligned base (128-byte swizzle atoms); the
  // dynamic window starts aligned in practice.  If it ever does not, report
  // and leave instead of computing on misaligned tiles.
  if (smem_u32(smem_split) & 1023u) {
    if (threadIdx.x == 0) atomicOr(status, 256);
    return;
  }
  const int kt = u.t[0];
  const int k0 = tile_orig(p, u, kt);
  const bool kvalid = u.part[0];

  uint8_t* smem = smem_split;
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBars + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const uint32_t sK = sb + L::kK, sV = sb + L::kV;
  auto sQ = [&](int st) { return sb + L::kQ + st * L::kTileBytes; };
  auto sdO = [&](int st) { return sb + L::kdO + st * L::kTileBytes; };
  auto sdS = [&](int x) { return sb + L::kdS + x * L::kHalfBytes; };
  auto sStat = [&](int st) { return sb + L::kStat + st * L::kStatBytes; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bar(KV_FULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(QD_FULL + i), 1);
      mbar_init(bar(QD_EMPTY + i), 1);
      mbar_init(bar(SP_FULL + i), 1);
      mbar_init(bar(DS_READY + i), 128);
      mbar_init(bar(DQ_FULL + i), 1);
      mbar_init(bar(DQ_FREE + i), 128);
      mbar_init(bar(RED_DONE + i), 2);
    }
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
  auto tS = [&](int x) { return tmem + 64 * x; };
  auto tDP = [&](int x) { return tmem + 128 + 64 * x; };
  const uint32_t tdV = tmem + 256, tdK = tmem + 384;
  const int row_base = u.b * p.N;
  const size_t stat_base = ((size_t)u.b * p.H + u.h) * p.N;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && kvalid) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(KV_FULL), 2 * L::kTileBytes);
      for (int c = 0; c < kChunks; ++c) {
        tma_load_3d(sK + c * kChunkBytes, &tmK, c * 64, u.h, row_base + k0, bar(KV_FULL));
        tma_load_3d(sV + c * kChunkBytes, &tmV, c * 64, u.h, row_base + k0, bar(KV_FULL));
      }
      int n = 0;
      bool ok = true;
      for (int qt = kt; ok && qt >= 0; qt = bwd::next_q(p, u, qt)) {
        const int st = n % kStages;
        if (n >= kStages) {  // MMAs done with the stage, and the dQ reductions staged in it have read it
          ok = s2_wait(bar(QD_EMPTY + st), ((n / kStages) - 1) & 1, abort_flag, status, 8);
          if (ok) ok = s2_wait(bar(RED_DONE + st), ((n / kStages) - 1) & 1, abort_flag, status, 8);
        }
        if (!ok) break;
        mbar_arrive_expect_tx(bar(QD_FULL + st), 2 * L::kTileBytes + L::kStatBytes);
        const int q0 = tile_orig(p, u, qt);
        for (int c = 0; c < kChunks; ++c) {
          tma_load_3d(sQ(st) + c * kChunkBytes, &tmQ, c * 64, u.h, row_base + q0, bar(QD_FULL + st));
          tma_load_3d(sdO(st) + c * kChunkBytes, &tmdO, c * 64, u.h, row_base + q0, bar(QD_FULL + st));
        }
        bulk_load(sStat(st), lse2 + stat_base + q0, kTile * 4, bar(QD_FULL + st));
        bulk_load(sStat(st) + kTile * 4, delta + stat_base + q0, kTile * 4, bar(QD_FULL + st));
        ++n;
      }
      for (int d = (n > kStages ? n - kStages : 0); d < n; ++d)
        s2_wait(bar(QD_FULL + d % kStages), (d / kStages) & 1, abort_flag, status, 8);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && kvalid) {
      constexpr uint32_t id_sp = umma_idesc_bf16(128, 64, 0, 0);   // S^T_x, dP^T_x
      constexpr uint32_t id_acc = umma_idesc_bf16(128, D, 0, 1);   // dV (A in TMEM), dK
      constexpr uint32_t id_dq = umma_idesc_bf16(128, 64, 1, 1);   // dQ^T_x = K^T dS^T_x
      bool ok = s2_wait(bar(KV_FULL), 0, abort_flag, status, 16);
      tc_fence_after();
      int n = 0;
      for (int qt = kt; ok && qt >= 0; qt = bwd::next_q(p, u, qt)) {
        const int st = n % kStages;
        ok = s2_wait(bar(QD_FULL + st), (n / kStages) & 1, abort_flag, status, 16);
        if (!ok) break;
        tc_fence_after();
        for (int x = 0; x < 2 && ok; ++x) {
          if (n > 0) {  // dQ^T_x(n-1) read out of the S columns, P^T_x(n-1) consumed
            ok = s2_wait(bar(DQ_FREE + x), (n - 1) & 1, abort_flag, status, 16);
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t qrow = x * 64 * 128;  // first query row of the half inside a 64-column chunk
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * kChunkBytes + (kk % 4) * 32;
            umma_ss(tS(x), umma_desc_sw128(sK + off, 16, 1024), umma_desc_sw128(sQ(st) + off + qrow, 16, 1024),
                    id_sp, kk > 0);
          }
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * kChunkBytes + (kk % 4) * 32;
            umma_ss(tDP(x), umma_desc_sw128(sV + off, 16, 1024), umma_desc_sw128(sdO(st) + off + qrow, 16, 1024),
                    id_sp, kk > 0);
          }
          umma_commit(bar(SP_FULL + x));
        }
        for (int x = 0; x < 2 && ok; ++x) {
          ok = s2_wait(bar(DS_READY + x), n & 1, abort_flag, status, 16);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qrow = x * 64 * 128;
          const bool first = (n == 0 && x == 0);
          // dV += P^T_x dO_x : K = 64 queries of the half
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tdV, tDP(x) + kk * 8, umma_desc_sw128(sdO(st) + qrow + kk * 2048, kChunkBytes, 1024), id_acc,
                    (!first || kk > 0) ? 1u : 0u);
          // dK += dS^T_x Q_x
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(tdK, umma_desc_sw128(sdS(x) + kk * 32, 16, 1024),
                    umma_desc_sw128(sQ(st) + qrow + kk * 2048, kChunkBytes, 1024), id_acc,
                    (!first || kk > 0) ? 1u : 0u);
          // dQ^T_x = K^T dS^T_x : M = D, K = 128 keys
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ss(tS(x), umma_desc_sw128(sK + kk * 2048, kChunkBytes, 1024),
                    umma_desc_sw128(sdS(x) + kk * 2048, kChunkBytes, 1024), id_dq, kk > 0 ? 1u : 0u);
          umma_commit(bar(DQ_FULL + x));
        }
        if (!ok) break;
        umma_commit(bar(QD_EMPTY + st));
        ++n;
      }
      umma_commit(bar(ACC_DONE));
      s2_wait(bar(ACC_DONE), 0, abort_flag, status, 16);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise warpgroups
    const int x = warp / 4;                 // query half [64x, 64x + 64)
    const int j = (warp % 4) * 32 + lane;   // key row == TMEM lane (also d for dQ^T)
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    bool ok = true;
    int n = 0;
    if (kvalid) {
      const bool key_tile_ragged = k0 + kTile > p.n_valid;
      const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
      for (int qt = kt; ok && qt >= 0; qt = bwd::next_q(p, u, qt)) {
        const int st = n % kStages;
        const int q0 = tile_orig(p, u, qt);
        // masks are needed on the diagonal tile and on a key tile with padding;
        // padded queries are zeroed by their -inf statistic
        const bool masked = (qt == kt) || key_tile_ragged;
        int lo = 0, hi = kTile;
        if (masked) query_range(p, u, kt, qt, j, lo, hi);
        // the stage's -lse2 / -Delta rows come with its Q/dO tiles
        ok = s2_wait(bar(QD_FULL + st), (n / kStages) & 1, abort_flag, status, 32);
        if (!ok) break;
        ok = s2_wait(bar(SP_FULL + x), n & 1, abort_flag, status, 32);
        if (!ok) break;
        tc_fence_after();
        const float2* nl = reinterpret_cast<const float2*>(smem + L::kStat + st * L::kStatBytes) + 32 * x;
        const float2* nd = nl + kTile / 2;
#pragma unroll
        for (int c = 0; c < 2; ++c) {  // 32 query columns per chunk
          uint32_t sv[32], dp[32];
          tmem_ld32(tS(x) + lane_off + 32 * c, sv);
          tmem_ld32(tDP(x) + lane_off + 32 * c, dp);
          tmem_wait_ld();
          uint32_t pp[16], dsp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            // P = 2^(S·log2(e)/sqrt(D) - lse·log2(e)),  dS = P (dP - Delta), two columns at a time
            const float2 a =
                __ffma2_rn(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), c2, nl[16 * c + i]);
            float p0 = ex2(a.x), p1 = ex2(a.y);
            if (masked) {
              const int col = 64 * x + 32 * c + 2 * i;
              p0 = (col >= lo && col < hi) ? p0 : 0.f;
              p1 = (col + 1 >= lo && col + 1 < hi) ? p1 : 0.f;
            }
            const float2 d2 =
                __fadd2_rn(make_float2(__uint_as_float(dp[2 * i]), __uint_as_float(dp[2 * i + 1])), nd[16 * c + i]);
            const float2 ds = __fmul2_rn(make_float2(p0, p1), d2);
            pp[i] = pack_bf16(p0, p1);
            dsp[i] = pack_bf16(ds.x, ds.y);
          }
          // P^T (bf16 pairs) into dP^T_x columns [16c, 16c + 16), already read
          tmem_st16(tDP(x) + lane_off + 16 * c, pp);
          // dS^T row j, queries [32c, 32c + 32): 16-byte pieces 4c..4c+3, 128-byte swizzle
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int piece = 4 * c + q;
            st_shared_v4(sdS(x) + j * 128 + ((piece ^ (j & 7)) << 4), dsp[4 * q], dsp[4 * q + 1], dsp[4 * q + 2],
                         dsp[4 * q + 3]);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(DS_READY + x));
        // dQ^T_x (lane = d, columns = the half's 64 queries): into registers, then
        // release the TMEM columns at once so the next S^T_x / dP^T_x can start
        ok = s2_wait(bar(DQ_FULL + x), n & 1, abort_flag, status, 32);
        if (!ok) break;
        tc_fence_after();
        uint32_t dq[64];
        tmem_ld32(tS(x) + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&dq[0]));
        tmem_ld32(tS(x) + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&dq[32]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(DQ_FREE + x));
        // Add into the fp32 accumulator with bulk tensor reductions, staged in this
        // half's rows [64x, 64x + 64) of the stage's Q and dO tiles: every MMA
        // reading them (S^T_x, dP^T_x, dV_x, dK_x) has completed at DQ_FULL[x], the
        // other half never reads them, and the producer refills the stage only
        // after RED_DONE.  Four 8 KB regions (Q and dO, 64-column chunks 0 and 1)
        // hold the eight 32 x 32 fp32 boxes: region b = d / 32, box row = query.
        const uint32_t region = ((j / 32) < 2 ? sQ(st) : sdO(st)) + ((j / 32) & 1) * kChunkBytes + x * 8192;
        const uint32_t stage_col = region + (j % 32) * 4;
#pragma unroll
        for (int q = 0; q < 64; ++q)
          st_shared_f32(stage_col + (q / 32) * 4096 + (q % 32) * 128, __uint_as_float(dq[q]));
        fence_proxy_async_smem();
        named_bar_sync(3 + x, 128);
        if (j == 0) {
          for (int b = 0; b < 4; ++b) {
            const uint32_t reg = (b < 2 ? sQ(st) : sdO(st)) + (b & 1) * kChunkBytes + x * 8192;
            for (int r = 0; r < 2; ++r)
              tma_reduce_add_3d(&tmdQacc, reg + r * 4096, 32 * b, u.h, row_base + q0 + 64 * x + 32 * r);
          }
          tma_store_commit();
          tma_store_wait_read();
          mbar_arrive(bar(RED_DONE + st));
        }
        ++n;
      }
      if (j == 0) tma_store_wait_all();  // every reduction has landed before the CTA retires
    }
    // the last reductions read Q stage rows the epilogue below overwrites
    named_bar_sync(1, 256);
    // ---------------------------------------------------------- epilogue: dK, dV
    bool have = kvalid && ok && n > 0;
    if (have) {
      have = s2_wait(bar(ACC_DONE), 0, abort_flag, status, 32);
      tc_fence_after();
    }
    const bool key_valid = have && (k0 + j < p.n_valid);
    const float scale = p.scale_log2 * 0.69314718055994531f;  // 1/sqrt(D)
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint32_t tsrc = which == 0 ? tdV : tdK;
      const float mul = which == 0 ? 1.f : scale;
      const uint32_t stage = sQ(which);
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const int d0 = x * 64 + 32 * c2;
        uint32_t v[32];
        if (have) {
          tmem_ld32(tsrc + lane_off + d0, v);
          tmem_wait_ld();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = d0 + 8 * q;
          const int chunk = col / 64, piece = (col % 64) / 8;
          uint32_t w[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float a = key_valid ? __uint_as_float(v[8 * q + 2 * t]) * mul : 0.f;
            const float b = key_valid ? __uint_as_float(v[8 * q + 2 * t + 1]) * mul : 0.f;
            w[t] = pack_bf16(a, b);
          }
          st_shared_v4(stage + chunk * kChunkBytes + j * 128 + ((piece ^ (j & 7)) << 4), w[0], w[1], w[2], w[3]);
        }
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 0) {
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
}

template <int D>
int launch_bwd_impl(const BwdArgs& a, int stages) {
  using L = bwd::Layout<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  const Plan& p = a.plan;
  const long long rows = (long long)p.B * p.N * p.H;
  cudaError_t e;
  if (stages & 1) {  // prepare: Delta, lse2, zeroed dq accumulator
    constexpr int kRowsPerBlock = 256 / (D / 8);
    s2_bwd_pre<D><<<(unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.lse, a.delta, a.lse2,
        p.B, p.N, p.H, p.n_valid);
    e = cudaMemsetAsync(a.dq_acc, 0, (size_t)rows * D * sizeof(float), a.stream);
    if (e != cudaSuccess) return (int)e;
  }
  if (stages & 2) {  // main: dK, dV and the dq accumulator
    const int grid = grid_bwd(p);
    if (D == 128) {
      static_assert(bwds::Layout::kBytes <= 232448, "shared memory budget");
      e = cudaFuncSetAttribute(s2_bwd_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bwds::Layout::kBytes);
      if (e != cudaSuccess) return (int)e;
      s2_bwd_split_kernel<<<grid, bwds::kThreads, bwds::Layout::kBytes, a.stream>>>(
          *a.tmQ, *a.tmK, *a.tmV, *a.tmdO, *a.tmdK, *a.tmdV, *a.tmdQacc, p, a.delta, a.lse2, a.status);
    } else {
      e = cudaFuncSetAttribute(s2_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
      if (e != cudaSuccess) return (int)e;
      s2_bwd_kernel<D><<<grid, bwd::kThreads, L::kAlloc, a.stream>>>(*a.tmQ, *a.tmK, *a.tmV, *a.tmdO, *a.tmdK,
                                                                     *a.tmdV, p, a.delta, a.lse2, a.dq_acc, a.status);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
  }
  if (stages & 4) {  // finish: dq = bf16(scale * accumulator)
    const long long n4 = rows * D / 4;
    const float scale = p.scale_log2 * 0.69314718055994531f;
    s2_bwd_dq_convert<<<148 * 8, 256, 0, a.stream>>>(reinterpret_cast<const float4*>(a.dq_acc),
                                                    static_cast<uint2*>(a.dq), n4, scale);
  }
  return (int)cudaGetLastError();
}

int launch_bwd(const BwdArgs& a, int stages) {
  if (a.plan.D == 64) return launch_bwd_impl<64>(a, stages);
  return launch_bwd_impl<128>(a, stages);
}

}  // namespace s2
