// s2_rope.cu -- rotary position prologue on original positions.
//
// "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 ("RoPE使用原始位置"): the
// shift only permutes tensors, so Q and K are rotated at each token's original
// position ID (never its index inside a group), and context extension maps a
// target position p to p·L0/L1 (position interpolation) before the angles are
// taken.  Pairing (the pages leave it open): coordinate k with k + D/2, the
// convention of the Llama models the pages fine-tune, with angle
// a_k = (p·scale)·base^(-2k/D):
//     x'[k] = x[k] cos a_k - x[k + D/2] sin a_k,  x'[k + D/2] = x[k + D/2] cos a_k + x[k] sin a_k.
//
// The pass is HBM-bound (read and write Q and K once), so it stays a separate
// kernel rather than a register pass inside the attention kernels, whose Q/K
// tiles go straight from TMA into the tensor cores' shared-memory layout.
// Angles reach 10^5 rad at the positions of long contexts, beyond fp32's
// resolution, so each (position, k) angle is formed and reduced in fp64 once
// per CTA and shared by all heads of Q and K at that position.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_kernels.h"

namespace s2 {

namespace {

constexpr int kRopeThreads = 256;

template <int D>
// q_out / k_out may alias q / k (in place): every thread reads its elements before writing them.
__global__ void __launch_bounds__(kRopeThreads) s2_rope_kernel(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                               __nv_bfloat16* q_out, __nv_bfloat16* k_out,
                                                               const int* __restrict__ positions, int B, int N,
                                                               int H, double base, double scale) {
  constexpr int kHalf = D / 2;
  constexpr int kPos = 2 * kRopeThreads / D;  // positions per CTA: one angle per thread
  __shared__ float2 cs[kPos][kHalf];          // (cos, sin)
  const long long row0 = (long long)blockIdx.x * kPos;  // flattened (b, n)
  const long long rows = (long long)B * N;
  {
    const int t = threadIdx.x, pr = t / kHalf, kk = t % kHalf;
    const long long row = row0 + pr;
    if (row < rows) {
      const long long pos = positions ? positions[row] : row % N;
      const double a = (double)pos * scale * pow(base, -2.0 * kk / D);
      double s, c;
      sincos(a, &s, &c);
      cs[pr][kk] = make_float2((float)c, (float)s);
    }
  }
  __syncthreads();
  // groups of 8 consecutive pairs: (head, k0) with k0 = 8m, m < kHalf/8
  constexpr int kGroups = kHalf / 8;
  const int per_row = H * kGroups;
  for (int w = threadIdx.x; w < kPos * 2 * per_row; w += kRopeThreads) {
    const int pr = w / (2 * per_row), rem = w % (2 * per_row);
    const int tensor = rem / per_row, g = rem % per_row;
    const long long row = row0 + pr;
    if (row >= rows) continue;
    const int h = g / kGroups, k0 = (g % kGroups) * 8;
    const size_t base_off = ((size_t)row * H + h) * D;
    const __nv_bfloat16* src = tensor ? k : q;
    __nv_bfloat16* dst = tensor ? k_out : q_out;
    const uint4 lo_raw = *reinterpret_cast<const uint4*>(src + base_off + k0);
    const uint4 hi_raw = *reinterpret_cast<const uint4*>(src + base_off + kHalf + k0);
    const __nv_bfloat162* lo2 = reinterpret_cast<const __nv_bfloat162*>(&lo_raw);
    const __nv_bfloat162* hi2 = reinterpret_cast<const __nv_bfloat162*>(&hi_raw);
    uint4 lo_out, hi_out;
    __nv_bfloat162* lo_o = reinterpret_cast<__nv_bfloat162*>(&lo_out);
    __nv_bfloat162* hi_o = reinterpret_cast<__nv_bfloat162*>(&hi_out);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 x = __bfloat1622float2(lo2[t]), y = __bfloat1622float2(hi2[t]);
      const float2 c0 = cs[pr][k0 + 2 * t], c1 = cs[pr][k0 + 2 * t + 1];
      lo_o[t] = __floats2bfloat162_rn(x.x * c0.x - y.x * c0.y, x.y * c1.x - y.y * c1.y);
      hi_o[t] = __floats2bfloat162_rn(y.x * c0.x + x.x * c0.y, y.y * c1.x + x.y * c1.y);
    }
    *reinterpret_cast<uint4*>(dst + base_off + k0) = lo_out;
    *reinterpret_cast<uint4*>(dst + base_off + kHalf + k0) = hi_out;
  }
}

}  // namespace

int launch_rope(const void* q, const void* k, void* q_out, void* k_out, const int* positions, int B, int N, int H,
                int D, double base, double scale, cudaStream_t stream) {
  const long long rows = (long long)B * N;
  const int per_cta = 2 * kRopeThreads / D;
  const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
  if (D == 64)
    s2_rope_kernel<64><<<grid, kRopeThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(q_out),
        static_cast<__nv_bfloat16*>(k_out), positions, B, N, H, base, scale);
  else
    s2_rope_kernel<128><<<grid, kRopeThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(q_out),
        static_cast<__nv_bfloat16*>(k_out), positions, B, N, H, base, scale);
  return (int)cudaGetLastError();
}

}  // namespace s2
