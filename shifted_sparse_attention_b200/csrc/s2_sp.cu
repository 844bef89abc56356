// s2_sp.cu -- halo movement of sequence-parallel S²-Attn.
//
// "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 (distributed boundaries):
// with the sequence cut into G-aligned shards, only the shifted heads cross a
// rank boundary, and they need the half group s = G/2 of K/V rows in front of
// the shard from the neighbouring rank; the backward returns the gradients of
// those rows the same way.  The volume per direction is 2·B·(H/2)·s·D
// elements, the pages' V_KV.
//
// A rank keeps every tensor in an extended buffer [B, s + L, H, D] whose rows
// [0, s) are the halo.  These kernels move the shifted heads' rows between
// such buffers and a packed message [2][B][s][H/2][D] (two tensors: K and V,
// or dK and dV), which the collective layer sends as one contiguous block:
//   pack   KV:   rows [L, L + s) (the shard's last s rows)  -> message
//   unpack KV:   message -> rows [0, s) (the halo)
//   pack   GRAD: rows [0, s) (the halo's partial gradients) -> message
//   unpack GRAD: rows [L, L + s) += message (summed in fp32, rounded once)
// 16-byte vectors, grid-stride over the message: an HBM-bound copy.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_kernels.h"

namespace s2 {

namespace {

constexpr int kHaloThreads = 256;

// One 16-byte vector (8 elements) per iteration; `pack` copies tensor rows
// into the message, otherwise the message goes into the tensors (added when
// `accumulate`).  row0: first tensor row (extended coordinates) of the halo.
__global__ void __launch_bounds__(kHaloThreads) s2_halo_kernel(__nv_bfloat16* a, __nv_bfloat16* b,
                                                               __nv_bfloat16* msg, int B, int Ne, int H, int D,
                                                               int s, int row0, bool pack, bool accumulate) {
  const int hh = H / 2, vec_per_row = hh * D / 8;  // vectors per (tensor, batch, halo row)
  const long long per_tensor = (long long)B * s * vec_per_row;
  const long long total = 2 * per_tensor;
  for (long long w = (long long)blockIdx.x * kHaloThreads + threadIdx.x; w < total;
       w += (long long)gridDim.x * kHaloThreads) {
    const int t = (int)(w / per_tensor);
    const long long r = w % per_tensor;
    const int bb = (int)(r / ((long long)s * vec_per_row));
    const long long r2 = r % ((long long)s * vec_per_row);
    const int e = (int)(r2 / vec_per_row), c = (int)(r2 % vec_per_row);
    // element offset of the vector in the tensor: row row0 + e, head H/2 + c / (D/8), column 8·(c % (D/8))
    const size_t off = (((size_t)bb * Ne + row0 + e) * H + hh) * D + (size_t)c * 8;
    __nv_bfloat16* x = t ? b : a;
    uint4* tv = reinterpret_cast<uint4*>(x + off);
    uint4* mv = reinterpret_cast<uint4*>(msg) + w;
    if (pack) {
      *mv = *tv;
    } else if (!accumulate) {
      *tv = *mv;
    } else {
      uint4 cur = *tv;
      const uint4 add = *mv;
      __nv_bfloat162* c2 = reinterpret_cast<__nv_bfloat162*>(&cur);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&add);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 u = __bfloat1622float2(c2[i]), v = __bfloat1622float2(a2[i]);
        c2[i] = __floats2bfloat162_rn(u.x + v.x, u.y + v.y);
      }
      *tv = cur;
    }
  }
}

}  // namespace

int launch_halo(void* a, void* b, void* msg, int B, int L, int H, int D, int G, int part, bool pack,
                cudaStream_t stream) {
  const int s = G / 2, Ne = s + L;
  // KV: the shard's last s rows travel to the next rank's halo;
  // GRAD: the halo's gradients travel back onto the previous rank's last s rows.
  const int row0 = (part == 0) == pack ? L : 0;
  const bool accumulate = part == 1 && !pack;
  const long long vecs = 2LL * B * s * (H / 2) * (D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (vecs + kHaloThreads - 1) / kHaloThreads;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  if (blocks < 1) blocks = 1;
  s2_halo_kernel<<<(unsigned)blocks, kHaloThreads, 0, stream>>>(
      static_cast<__nv_bfloat16*>(a), static_cast<__nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(msg), B, Ne, H, D,
      s, row0, pack, accumulate);
  return (int)cudaGetLastError();
}

}  // namespace s2
