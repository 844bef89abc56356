// s2_kernels.h -- internal launch interface between the C-ABI layer and the
// kernels (not installed; the public interface is include/s2attn.h).
#pragma once
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "s2_index.cuh"

namespace s2 {

struct FwdArgs {
  const CUtensorMap* tmQ;
  const CUtensorMap* tmK;
  const CUtensorMap* tmV;
  const CUtensorMap* tmO;
  Plan plan;
  float* lse;
  int* status;
  cudaStream_t stream;
};

struct BwdArgs {
  const CUtensorMap* tmQ;
  const CUtensorMap* tmK;
  const CUtensorMap* tmV;
  const CUtensorMap* tmdO;
  const CUtensorMap* tmdK;
  const CUtensorMap* tmdV;
  const CUtensorMap* tmdQ;
  Plan plan;
  const void* o;      // bf16 [B, N, H, D]
  const void* dout;   // bf16 [B, N, H, D]
  const float* lse;   // [B, H, N]
  float* delta;       // workspace [B, H, N]: -(dout_i·o_i)
  float* lse2;        // workspace [B, H, N]: -lse_i·log2(e), -inf on padded rows
  void* ds;           // stored-dS workspace (bf16 tiles of 32 KB, see s2_index.cuh), or null
  int* status;
  cudaStream_t stream;
};

int launch_fwd(const FwdArgs& a);
// stages: 1 = prepare (Delta, lse2), 2 = dK/dV pass, 4 = dQ pass; with 8 the
// dK/dV pass also stores dS and the dQ pass reads it instead of recomputing.
int launch_bwd(const BwdArgs& a, int stages);
// Sets the calling thread's s2attn_last_error() message; returns `code`.
int report_error(int code, const char* fmt, ...);
// Process-unique ID of the calling thread's current CUDA context (0 if unknown):
// per-device caches of device addresses are valid only inside that context.
unsigned long long current_context_id();

int launch_adjacency(const Plan& p, int head_class, int format, void* out, cudaStream_t stream);
// Failure-detection probe: a bounded wait on a barrier nothing completes.
int launch_wait_probe(int* status, long long budget, cudaStream_t stream);
int launch_bounds_probe(int* status, long long v, long long lo, long long hi, cudaStream_t stream);

// Training / inference graph gap: per-row rho and output shift, per (head
// class, bucket) statistics float32 [2][kGapBuckets][4].
constexpr int kGapBuckets = 32;
int launch_graph_gap(const Plan& p, const float* lse_s, const float* lse_f, const void* o_s, const void* o_f,
                     float* rho, float* dist, float* stats, cudaStream_t stream);

// Halo movement of sequence-parallel ranks (part 0: K/V, 1: gradients; pack:
// tensors -> message, else message -> tensors, accumulated for gradients).
int launch_halo(void* a, void* b, void* msg, int B, int L, int H, int D, int G, int part, bool pack,
                cudaStream_t stream);

// Rotary position prologue on original positions (positions: int32 [B, N] or null = 0..N-1).
int launch_rope(const void* q, const void* k, void* q_out, void* k_out, const int* positions, int B, int N, int H,
                int D, double base, double scale, cudaStream_t stream);

// Per-position document bounds [B, N, 2] from per-position document IDs [B, N].
int launch_doc_bounds(const int32_t* ids, int32_t* bounds, int B, int N, cudaStream_t stream);

}  // namespace s2
