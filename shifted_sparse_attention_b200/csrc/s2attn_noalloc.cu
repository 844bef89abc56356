// s2attn_noalloc.cu -- the backward for callers that cannot allocate device
// memory themselves.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they need the backward: for example a plug-in running inside a
// host framework that owns the whole device heap and forbids third-party
// allocations, or a runtime that must keep a fixed, pre-planned memory
// footprint.  They can still pass their inputs and outputs, but not the
// backward's scratch workspace.  s2attn_bwd_noalloc_v gives them the same
// backward with its scratch taken from a fixed array that lives in this
// library's device image.
//
// The array is a file-scope __device__ variable of kScratchBytes (32 MiB):
// every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address, so on the first call
// on each device (with that device current) the address is looked up once
// with cudaGetSymbolAddress and cached; that first call should therefore be
// made before any stream capture starts.  Every call shares the one array, so
// calls whose kernels overlap on the GPU (different streams, or different
// host threads on one device) race on it.  The array keeps whatever the last
// call left in it; the backward's prepare stage rewrites every row statistic
// the later stages read, so nothing has to be cleared.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/s2attn.h"
#include "s2_kernels.h"

namespace {

constexpr size_t kScratchBytes = S2_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes == (size_t(32) << 20), "scratch size is part of the documented ABI");

static __device__ __align__(256) unsigned char g_s2_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

}  // namespace

extern "C" int s2attn_bwd_noalloc_v(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                    const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H,
                                    int64_t D, int64_t G, int64_t n_valid, int variant, void* stream) {
  const size_t need = s2attn_bwd_workspace_size(B, N, H, D);
  if (need == 0) return s2::report_error(S2_ERR_SHAPE, "B, N, H, D must be positive");
  if (need > kScratchBytes)
    return s2::report_error(S2_ERR_UNSUPPORTED,
                            "s2attn_bwd_noalloc_v: this shape needs %zu bytes of scratch, more than the fixed %zu "
                            "(use s2attn_bwd_v with a caller-provided workspace)",
                            need, kScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return s2::report_error(S2_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return s2::report_error(S2_ERR_UNSUPPORTED, "device index %d out of range", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
      e = cudaSetDevice(dev);  // the device must be current for the symbol lookup
      if (e != cudaSuccess) return s2::report_error(S2_ERR_CUDA, "cudaSetDevice: %s", cudaGetErrorString(e));
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_s2_noalloc_scratch);
      if (e != cudaSuccess || addr == nullptr)
        return s2::report_error(S2_ERR_CUDA, "cudaGetSymbolAddress of the scratch array: %s", cudaGetErrorString(e));
      g_scratch_addr[dev] = addr;
    }
    scratch = g_scratch_addr[dev];
  }
  return s2attn_bwd_stages_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, n_valid, variant, scratch,
                             kScratchBytes, S2_BWD_ALL, stream);
}
