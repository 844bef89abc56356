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
// The array is a file-scope __device__ variable of kScratchBytes (32 MiB).
// The driver reserves it when it loads this file's device module into a
// context: with CUDA's default lazy module loading that happens inside the
// first call on each device (at the symbol lookup below), with
// CUDA_MODULE_LOADING=EAGER when the context is created.  It then stays
// reserved until the context is destroyed.  A caller whose framework will
// later claim the device heap should therefore make one call at start-up,
// before the framework reserves its memory; if the device has no 32 MiB left
// at that first call, the lookup fails and the call returns S2_ERR_CUDA with
// the driver's out-of-memory message.
//
// Host code cannot use the array's name as a device address, so the first
// call on each device (with that device current) looks the address up with
// cudaGetSymbolAddress and caches it together with the identity of the
// context it belongs to; a later call in another context of that device (for
// example after cudaDeviceReset) looks it up again.  The first call should
// be made before any stream capture starts.  Every call shares the one array,
// so calls whose kernels overlap on the GPU (different streams, or different
// host threads on one device) race on it.  The array keeps whatever the last
// call left in it; the backward's prepare stage rewrites every row statistic
// the later stages read, so nothing has to be cleared.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/s2attn.h"
#include "s2_kernels.h"

namespace {

constexpr size_t kScratchBytes = S2_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes == (size_t(32) << 20), "scratch size is part of the documented ABI");

static __device__ __align__(256) unsigned char g_s2_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct Cached {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;  // context the address belongs to
};
Cached g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

int cuda_fail(cudaError_t e, const char* what) {
  cudaGetLastError();  // leave no sticky-looking error behind for the caller's next check
  return s2::report_error(S2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

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
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return s2::report_error(S2_ERR_UNSUPPORTED, "device index %d out of range", dev);
  // the same capability rule as every other entry point, before the module (and its
  // array) is loaded: on another GPU the lookup would fail for want of a kernel image
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10 || minor != 0)
    return s2::report_error(S2_ERR_UNSUPPORTED, "kernels are built for sm_100a (B200); device is sm_%d%d", major,
                            minor);
  e = cudaSetDevice(dev);  // the device's primary context must be current for the symbol lookup
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  const unsigned long long ctx = s2::current_context_id();
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    Cached& c = g_scratch[dev];
    if (!c.addr || (ctx != 0 && c.ctx_id != ctx)) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_s2_noalloc_scratch);
      if (e != cudaSuccess || addr == nullptr)
        return cuda_fail(e, "cudaGetSymbolAddress of the 32 MiB scratch array (reserved when the module loads)");
      c.addr = addr;
      c.ctx_id = ctx;
    }
    scratch = c.addr;
  }
  return s2attn_bwd_stages_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, n_valid, variant, scratch,
                             kScratchBytes, S2_BWD_ALL, stream);
}
