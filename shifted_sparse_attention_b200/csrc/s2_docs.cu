// s2_docs.cu -- document bounds for packed sequences.
//
// "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 (packing): several
// documents packed into one sequence need a document mask in both the
// original and the shifted grouping.  The attention kernels take, for every
// position, the bounds [first, one past last] of its document (original
// positions); this kernel derives them from per-position document IDs, a
// document being a maximal run of equal IDs.
//
// One CTA per batch row.  Each thread owns a contiguous chunk of positions:
// it finds the last run start and the first run end inside its chunk, a
// block-wide scan carries them across chunks (prefix maximum of starts,
// suffix minimum of ends), and a second pass over the chunk writes the bounds.
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "s2_kernels.h"

namespace s2 {

namespace {

constexpr int kDocThreads = 1024;

__global__ void __launch_bounds__(kDocThreads) s2_doc_bounds_kernel(const int32_t* __restrict__ ids,
                                                                    int32_t* __restrict__ bounds, int N) {
  __shared__ int s_start[kDocThreads];
  __shared__ int s_end[kDocThreads];
  const int b = blockIdx.x, t = threadIdx.x;
  const int32_t* id = ids + (size_t)b * N;
  int32_t* out = bounds + (size_t)b * N * 2;
  const int chunk = (N + kDocThreads - 1) / kDocThreads;
  const int lo = t * chunk < N ? t * chunk : N;
  const int hi = lo + chunk < N ? lo + chunk : N;

  // run boundaries inside the chunk: x starts a run if x == 0 or id[x] != id[x-1];
  // x ends a run (its end bound is x + 1) if x == N-1 or id[x] != id[x+1]
  int last_start = -1, first_end = INT_MAX;
  for (int x = lo; x < hi; ++x)
    if (x == 0 || id[x] != id[x - 1]) last_start = x;
  for (int x = hi - 1; x >= lo; --x)
    if (x == N - 1 || id[x] != id[x + 1]) first_end = x + 1;
  s_start[t] = last_start;
  s_end[t] = first_end;
  __syncthreads();
  // inclusive prefix maximum of starts and suffix minimum of ends over the chunks
  for (int off = 1; off < kDocThreads; off <<= 1) {
    const int a = t >= off ? s_start[t - off] : -1;
    const int e = t + off < kDocThreads ? s_end[t + off] : INT_MAX;
    __syncthreads();
    if (a > s_start[t]) s_start[t] = a;
    if (e < s_end[t]) s_end[t] = e;
    __syncthreads();
  }
  int cur = t > 0 ? s_start[t - 1] : -1;  // start of the run that is open when the chunk begins
  for (int x = lo; x < hi; ++x) {
    if (x == 0 || id[x] != id[x - 1]) cur = x;
    out[2 * (size_t)x] = cur;
  }
  cur = t + 1 < kDocThreads ? s_end[t + 1] : INT_MAX;  // end of the run still open after the chunk
  for (int x = hi - 1; x >= lo; --x) {
    if (x == N - 1 || id[x] != id[x + 1]) cur = x + 1;
    out[2 * (size_t)x + 1] = cur;
  }
}

}  // namespace

int launch_doc_bounds(const int32_t* ids, int32_t* bounds, int B, int N, cudaStream_t stream) {
  s2_doc_bounds_kernel<<<B, kDocThreads, 0, stream>>>(ids, bounds, N);
  return (int)cudaGetLastError();
}

}  // namespace s2
