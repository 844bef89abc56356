// s2_adj.cu -- debug dump of the visibility pattern the kernels actually use.
//
// Walks the same work-unit decomposition (decode_unit), the same key-tile
// list (ktile_valid / tile_takes) and the same per-row column limits
// (col_limit) as the forward and backward kernels, and writes, for every
// query row of one head class, the set of keys those kernels visit, in
// original positions.  Comparing it bit for bit with the explicit matrices
// A^(0) / A^(1) of "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1 checks the
// scheduler and the masks independently of any floating-point result.
#include <cuda_runtime.h>

#include "s2_debug.cuh"
#include "s2_index.cuh"
#include "s2_kernels.h"
#include "sm100_ptx.cuh"

namespace s2 {

// One CTA per work unit of a head of class `cls`; thread = one row of the
// unit's two query tiles.  With a document mask (p.docs, one batch row) the
// walk is the document-aware forward's: query tiles that hold a valid row,
// key tiles that meet the span of the query tile's documents, and each row's
// columns clipped to its document.
__global__ void __launch_bounds__(256) s2_adjacency_kernel(const __grid_constant__ Plan p, int cls, int format,
                                                           uint32_t* __restrict__ bits,
                                                           int* __restrict__ intervals) {
  Unit u;
  if (!decode_unit(p, blockIdx.x, u)) return;
  if (u.h != cls) return;  // with H = 2, head h has class h (dense: only head 0 is dumped)
  const int x = threadIdx.x / kTile, r = threadIdx.x % kTile;
  if (u.t[x] < 0) return;
  const int row = tile_orig(p, u, u.t[x]) + r;
  const int words = (p.N + 31) / 32;
  if (format == 0)
    for (int w = 0; w < words; ++w) bits[(size_t)row * words + w] = 0u;
  int iv[4] = {-1, -1, -1, -1};
  int nint = 0;
  // under a document mask: the forward's tile test (the span of the documents
  // touching the query tile) and its per-row column range (row_cols)
  int dlo = 0, dhi = p.N;
  if (p.docs && u.part[x]) doc_span(p, u.b, tile_orig(p, u, u.t[x]), dlo, dhi);
  for (int k = 0; k <= u.t[x]; ++k) {
    if (!ktile_valid(p, u, k)) continue;
    int c0 = 0, c1 = 0;
    if (p.docs) {
      if (!u.part[x] || !tile_meets(tile_orig(p, u, k), dlo, dhi)) continue;
      row_cols(p, u, u.t[x], k, r, c0, c1);
    } else {
      if (!tile_takes(p, u, x, k)) continue;
      c1 = col_limit(p, u, u.t[x], k, r);
    }
    if (c1 <= c0) continue;
    const int lo = tile_orig(p, u, k) + c0, hi = tile_orig(p, u, k) + c1 - 1;
    if (format == 0) {
      for (int j = lo; j <= hi; ++j) bits[(size_t)row * words + j / 32] |= 1u << (j % 32);
    } else {
      if (nint > 0 && iv[2 * (nint - 1) + 1] + 1 == lo) {
        iv[2 * (nint - 1) + 1] = hi;
      } else if (nint < 2) {
        iv[2 * nint] = lo;
        iv[2 * nint + 1] = hi;
        ++nint;
      } else {
        iv[0] = iv[1] = iv[2] = iv[3] = -2;  // more than two intervals: never expected
      }
    }
  }
  if (format == 1)
    for (int c = 0; c < 4; ++c) intervals[(size_t)row * 4 + c] = iv[c];
}

__global__ void s2_fill_kernel(int* out, size_t n, int value) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    out[i] = value;
}

int launch_adjacency(const Plan& p0, int head_class, int format, void* out, cudaStream_t stream) {
  // A head of each class: with H = 2, head 0 is class 0 and head 1 is class 1.
  Plan p = p0;
  p.B = 1;
  p.H = 2;
  // rows that no tile covers cannot exist, but start from a defined state
  if (format == 1)
    s2_fill_kernel<<<64, 256, 0, stream>>>(static_cast<int*>(out), (size_t)p.N * 4, -1);
  const int grid = grid_fwd(p);
  s2_adjacency_kernel<<<grid, 256, 0, stream>>>(p, head_class, format, static_cast<uint32_t*>(out),
                                                static_cast<int*>(out));
  return (int)cudaGetLastError();
}

// Failure-detection probe: the kernels' bounded-wait path, exercised without a
// fault.  Two warps of one CTA wait on an mbarrier that nothing completes:
// warp 0 with a short clock budget -- it gives up, raises the CTA's abort flag
// and records bit 512 in the status word, as a kernel role does on a timeout;
// warp 1 with the kernels' own bounded wait, which returns as soon as the flag
// is up.  The CTA then exits normally and the context stays usable.
__global__ void s2_wait_probe_kernel(int* __restrict__ status, long long budget) {
  __shared__ alignas(8) uint64_t bar_word;
  __shared__ int abort_word;
  const uint32_t b = smem_u32(&bar_word);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    while (!mbar_try_wait(b, 0)) {
      if (clock64() - t0 > budget) {
        *reinterpret_cast<volatile int*>(&abort_word) = 1;
        atomicOr(status, 512);
        break;
      }
    }
  } else if (threadIdx.x == 32) {
    s2_wait(b, 0, reinterpret_cast<volatile int*>(&abort_word), status, 1024);
  }
  __syncthreads();
}

int launch_wait_probe(int* status, long long budget, cudaStream_t stream) {
  s2_wait_probe_kernel<<<1, 64, 0, stream>>>(status, budget);
  return (int)cudaGetLastError();
}

// One thread runs the kernels' bounds check on a value the caller chose.  No
// memory access depends on the outcome: this exercises the recording path
// (first violation wins, later ones only set the flag) without any fault.
__global__ void s2_bounds_probe_kernel(int* __restrict__ status, long long v, long long lo, long long hi) {
  (void)S2_IN(kSiteProbe, v, lo, hi);
}

int launch_bounds_probe(int* status, long long v, long long lo, long long hi, cudaStream_t stream) {
  s2_bounds_probe_kernel<<<1, 1, 0, stream>>>(status, v, lo, hi);
  return (int)cudaGetLastError();
}

}  // namespace s2
