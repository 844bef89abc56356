// s2_gap.cu -- the training / inference graph gap of S²-Attn.
//
// "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §3 ("稀疏训练与full推理之间的目标
// 偏移"): training normalises each row's softmax over its S² visible set S_i,
// inference over the full causal history F_i.  With Z_s the unnormalised
// mass inside S_i and Z_out the mass of F_i \ S_i, every in-group weight is
// scaled by Z_s / (Z_s + Z_out) when the graph switches.  From the two
// forwards' log-sum-exps that factor is rho_i = exp(lse_i^{S²} - lse_i^{full})
// (exactly Z_s / (Z_s + Z_out) when S_i ⊂ F_i, i.e. for the strict variant);
// the output shift is d_i = ||o_i^{S²} - o_i^{full}||_2.  §2.1 asks for such
// diagnostics bucketed by the query's distance to its group boundary: here a
// row's bucket is floor(log2(l + 1)) of its position l inside its S² segment.
//
// Two kernels: s2_gap_rows (one warp per row: rho and d) and s2_gap_stats
// (one CTA per (head class, bucket): count, mean rho, min rho, mean d, summed
// in a fixed order, so the statistics are deterministic).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_index.cuh"
#include "s2_kernels.h"

namespace s2 {

namespace {

constexpr int kGapThreads = 256;

// Bucket floor(log2(l + 1)) of original row x, l its position inside its S²
// segment (head class cls).
__device__ __forceinline__ int row_bucket(const Plan& p, int cls, int x) {
  const int v = virt_of(p, cls, x);
  int vb, len;
  seg_bounds(p, cls, seg_of(p, cls, v), vb, len);
  const unsigned l1 = (unsigned)(v - vb) + 1u;
  return 31 - __clz(l1);
}

__global__ void __launch_bounds__(kGapThreads) s2_gap_rows(const __grid_constant__ Plan p, const float* __restrict__ lse_s,
                                                           const float* __restrict__ lse_f,
                                                           const __nv_bfloat16* __restrict__ o_s,
                                                           const __nv_bfloat16* __restrict__ o_f,
                                                           float* __restrict__ rho, float* __restrict__ dist) {
  const long long row = (long long)blockIdx.x * (kGapThreads / 32) + threadIdx.x / 32;  // (b, h, i) in [B, H, N]
  const int lane = threadIdx.x % 32;
  const long long rows = (long long)p.B * p.H * p.N;
  if (row >= rows) return;
  const int i = (int)(row % p.N);
  const long long bh = row / p.N;
  const int h = (int)(bh % p.H), b = (int)(bh / p.H);
  // squared output difference, D / 32 elements per lane
  float acc = 0.f;
  const size_t base = (((size_t)b * p.N + i) * p.H + h) * p.D;
  for (int d = lane; d < p.D; d += 32) {
    const float e = __bfloat162float(o_s[base + d]) - __bfloat162float(o_f[base + d]);
    acc = fmaf(e, e, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const bool valid = i < p.n_valid;
    rho[row] = valid ? __expf(lse_s[row] - lse_f[row]) : 0.f;
    dist[row] = valid ? sqrtf(acc) : 0.f;
  }
}

// stats[(cls * kGapBuckets + k) * 4 + {0,1,2,3}] = {count, mean rho, min rho, mean d}
__global__ void __launch_bounds__(kGapThreads) s2_gap_stats(const __grid_constant__ Plan p, const float* __restrict__ rho,
                                                            const float* __restrict__ dist,
                                                            float* __restrict__ stats) {
  const int cls = blockIdx.x / kGapBuckets, k = blockIdx.x % kGapBuckets;
  const long long rows = (long long)p.B * p.H * p.N;
  double n = 0.0, sr = 0.0, sd = 0.0;
  float mn = INFINITY;
  for (long long row = threadIdx.x; row < rows; row += kGapThreads) {
    const int i = (int)(row % p.N), h = (int)((row / p.N) % p.H);
    if (i >= p.n_valid || head_class(p, h) != cls || row_bucket(p, cls, i) != k) continue;
    n += 1.0;
    sr += rho[row];
    sd += dist[row];
    mn = fminf(mn, rho[row]);
  }
  __shared__ double s_n[kGapThreads], s_r[kGapThreads], s_d[kGapThreads];
  __shared__ float s_m[kGapThreads];
  s_n[threadIdx.x] = n;
  s_r[threadIdx.x] = sr;
  s_d[threadIdx.x] = sd;
  s_m[threadIdx.x] = mn;
  __syncthreads();
  for (int off = kGapThreads / 2; off > 0; off >>= 1) {
    if ((int)threadIdx.x < off) {
      s_n[threadIdx.x] += s_n[threadIdx.x + off];
      s_r[threadIdx.x] += s_r[threadIdx.x + off];
      s_d[threadIdx.x] += s_d[threadIdx.x + off];
      s_m[threadIdx.x] = fminf(s_m[threadIdx.x], s_m[threadIdx.x + off]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    float* out = stats + (size_t)blockIdx.x * 4;
    const double c = s_n[0];
    out[0] = (float)c;
    out[1] = c > 0 ? (float)(s_r[0] / c) : 0.f;
    out[2] = c > 0 ? s_m[0] : 0.f;
    out[3] = c > 0 ? (float)(s_d[0] / c) : 0.f;
  }
}

}  // namespace

int launch_graph_gap(const Plan& p, const float* lse_s, const float* lse_f, const void* o_s, const void* o_f,
                     float* rho, float* dist, float* stats, cudaStream_t stream) {
  const long long rows = (long long)p.B * p.H * p.N;
  const long long blocks = (rows + kGapThreads / 32 - 1) / (kGapThreads / 32);
  s2_gap_rows<<<(unsigned)blocks, kGapThreads, 0, stream>>>(p, lse_s, lse_f,
                                                            static_cast<const __nv_bfloat16*>(o_s),
                                                            static_cast<const __nv_bfloat16*>(o_f), rho, dist);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  s2_gap_stats<<<2 * kGapBuckets, kGapThreads, 0, stream>>>(p, rho, dist, stats);
  return (int)cudaGetLastError();
}

}  // namespace s2
