// s2attn_api.cu -- the C ABI declared in include/s2attn.h: argument and shape
// validation (divisibility rules of "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调"
// §1: H even, G even, N a multiple of G; padding carried as n_valid), TMA
// tensor-map encoding, and kernel launches.  No device memory is allocated
// here; the only mutable state is a per-device cache (capability check,
// timeout status word address, driver entry point).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/s2attn.h"
#include "s2_debug.cuh"
#include "s2_index.cuh"
#include "s2_kernels.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

// Status area written by the kernels: [0] flag bits (timeouts per role, and
// the debug build's bounds flag), then the debug build's first bounds
// violation (s2_debug.cuh).
__device__ int g_s2_status[s2::kStatusInts];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
  bool ready = false;
  bool supported = false;
  int* status = nullptr;
  unsigned long long ctx_id = 0;  // context `status` belongs to
  EncodeTiledFn encode = nullptr;
  std::string why;
};

constexpr int kMaxDevices = 64;
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

// Per-device set-up on first use: capability check and the status word address.
int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(S2_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(S2_ERR_UNSUPPORTED, "device index %d out of range", dev);
  // Make the device's primary context current on this thread (callers such as
  // autograd worker threads may not have touched the runtime yet).
  e = cudaSetDevice(dev);
  if (e != cudaSuccess) return fail(S2_ERR_CUDA, "cudaSetDevice: %s", cudaGetErrorString(e));
  const unsigned long long ctx = s2::current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  // a new context of the device (e.g. after cudaDeviceReset) reloads the module:
  // the status word's address must be looked up again
  if (st.ready && st.supported && ctx != 0 && st.ctx_id != ctx) st.ready = false;
  if (!st.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return fail(S2_ERR_CUDA, "cudaGetDeviceProperties: %s", cudaGetErrorString(e));
    if (prop.major != 10 || prop.minor != 0) {
      st.supported = false;
      st.why = "kernels are built for sm_100a (B200); device is sm_" + std::to_string(prop.major) +
               std::to_string(prop.minor);
    } else {
      void* sym = nullptr;
      e = cudaGetSymbolAddress(&sym, g_s2_status);
      if (e != cudaSuccess) return fail(S2_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      st.status = static_cast<int*>(sym);
      st.ctx_id = ctx;
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(S2_ERR_CUDA, "driver entry point cuTensorMapEncodeTiled unavailable");
      st.encode = reinterpret_cast<EncodeTiledFn>(fn);
      st.supported = true;
    }
    st.ready = true;
  }
  if (!st.supported) return fail(S2_ERR_UNSUPPORTED, "%s", st.why.c_str());
  *out = &st;
  return S2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


// Shape rules of the method plus the kernels' own support limits.
int validate(int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant) {
  if (variant < S2_STRICT || variant > S2_DENSE_CAUSAL)
    return fail(S2_ERR_INVALID_ARG, "unknown variant %d", variant);
  if (B < 1 || N < 1 || H < 1 || D < 1 || G < 1)
    return fail(S2_ERR_SHAPE, "B, N, H, D, G must be positive (B=%lld N=%lld H=%lld D=%lld G=%lld)",
                (long long)B, (long long)N, (long long)H, (long long)D, (long long)G);
  if (H % 2) return fail(S2_ERR_SHAPE, "H=%lld must be even (half the heads are shifted)", (long long)H);
  if (G % 2) return fail(S2_ERR_SHAPE, "G=%lld must be even (shift G/2)", (long long)G);
  if (N % G) return fail(S2_ERR_SHAPE, "N=%lld must be a multiple of G=%lld (pad first)", (long long)N, (long long)G);
  if (n_valid < 1 || n_valid > N)
    return fail(S2_ERR_SHAPE, "n_valid=%lld must be in [1, N=%lld]", (long long)n_valid, (long long)N);
  if (D != 64 && D != 128) return fail(S2_ERR_UNSUPPORTED, "D=%lld: kernels support D in {64, 128}", (long long)D);
  if (variant == S2_DENSE_CAUSAL) {
    if (N % s2::kTile) return fail(S2_ERR_UNSUPPORTED, "N=%lld must be a multiple of 128", (long long)N);
  } else if ((G / 2) % s2::kTile) {
    return fail(S2_ERR_UNSUPPORTED, "G/2=%lld must be a multiple of 128", (long long)(G / 2));
  }
  if (B * N >= (int64_t(1) << 31) || B * H * N >= (int64_t(1) << 31))
    return fail(S2_ERR_UNSUPPORTED, "B*N and B*H*N must be below 2^31");
  return S2_OK;
}

int make_tmap(DeviceState* st, CUtensorMap* m, const void* base, int64_t B, int64_t N, int64_t H, int64_t D,
              int box_rows = s2::kTile) {
  // [B*N, H, D] bf16 viewed as a 3-D tensor (D innermost); box = 64 columns x 1 head x box_rows rows.
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(B * N)};
  cuuint64_t strides[2] = {(cuuint64_t)(D * 2), (cuuint64_t)(H * D * 2)};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t elem[3] = {1, 1, 1};
  CUresult r = st->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                          elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(S2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return S2_OK;
}

int launch_status(int rc, const char* what) {
  if (rc == 0) return S2_OK;
  return fail(S2_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString((cudaError_t)rc));
}

}  // namespace

namespace s2 {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Records a message for s2attn_last_error() from other translation units.
int report_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}
}  // namespace s2

extern "C" {

int s2attn_version(void) { return 201; }

const char* s2attn_last_error(void) { return g_last_error.c_str(); }

// Pointer checks, tensor maps over [B, plan.N, H, D] and the forward launch.
static int fwd_launch(const void* q, const void* k, const void* v, void* o, float* lse, const s2::Plan& plan,
                      void* stream) {
  int rc;
  const int64_t B = plan.B, N = plan.N, H = plan.H, D = plan.D;
  if (!q || !k || !v || !o || !lse) return fail(S2_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return fail(S2_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  CUtensorMap tq, tk, tv, to;
  if ((rc = make_tmap(st, &tq, q, B, N, H, D)) || (rc = make_tmap(st, &tk, k, B, N, H, D)) ||
      (rc = make_tmap(st, &tv, v, B, N, H, D)) || (rc = make_tmap(st, &to, o, B, N, H, D)))
    return rc;
  s2::FwdArgs a;
  a.tmQ = &tq; a.tmK = &tk; a.tmV = &tv; a.tmO = &to;
  a.plan = plan;
  a.lse = lse;
  a.status = st->status;
  a.stream = static_cast<cudaStream_t>(stream);
  return launch_status(s2::launch_fwd(a), "forward");
}

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* docs,
                    int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                    void* stream) {
  int rc = validate(B, N, H, D, G, n_valid, variant);
  if (rc) return rc;
  s2::Plan plan = s2::make_plan((int)B, (int)N, (int)H, (int)D, (int)G, (int)n_valid, variant);
  plan.docs = docs;
  return fwd_launch(q, k, v, o, lse, plan, stream);
}

int s2attn_fwd_v(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N,
                 int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant, void* stream) {
  return fwd_impl(q, k, v, o, lse, nullptr, B, N, H, D, G, n_valid, variant, stream);
}

int s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N,
               int64_t H, int64_t D, int64_t G, int variant, void* stream) {
  return s2attn_fwd_v(q, k, v, o, lse, B, N, H, D, G, N, variant, stream);
}

int s2attn_fwd_docs(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* doc_bounds,
                    int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                    void* stream) {
  if (!doc_bounds) return fail(S2_ERR_INVALID_ARG, "null doc_bounds (use s2attn_fwd_v without documents)");
  if (reinterpret_cast<uintptr_t>(doc_bounds) & 7u) return fail(S2_ERR_INVALID_ARG, "doc_bounds must be 8-byte aligned");
  return fwd_impl(q, k, v, o, lse, doc_bounds, B, N, H, D, G, n_valid, variant, stream);
}

int s2attn_graph_gap(const float* lse_s2, const float* lse_full, const void* o_s2, const void* o_full, int64_t B,
                     int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant, float* rho, float* dist,
                     float* stats, void* stream) {
  int rc = validate(B, N, H, D, G, n_valid, variant);
  if (rc) return rc;
  if (variant == S2_DENSE_CAUSAL) return fail(S2_ERR_INVALID_ARG, "variant must be the S² graph (strict or rolled)");
  if (!lse_s2 || !lse_full || !o_s2 || !o_full || !rho || !dist || !stats)
    return fail(S2_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(o_s2) || !aligned16(o_full) || (reinterpret_cast<uintptr_t>(lse_s2) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse_full) & 3u) || (reinterpret_cast<uintptr_t>(rho) & 3u) ||
      (reinterpret_cast<uintptr_t>(dist) & 3u) || (reinterpret_cast<uintptr_t>(stats) & 3u))
    return fail(S2_ERR_INVALID_ARG, "misaligned pointer");
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  const s2::Plan p = s2::make_plan((int)B, (int)N, (int)H, (int)D, (int)G, (int)n_valid, variant);
  return launch_status(
      s2::launch_graph_gap(p, lse_s2, lse_full, o_s2, o_full, rho, dist, stats, static_cast<cudaStream_t>(stream)),
      "graph gap");
}

int s2attn_rope(const void* q, const void* k, void* q_out, void* k_out, const int32_t* positions, int64_t B,
                int64_t N, int64_t H, int64_t D, double base, double scale, void* stream) {
  if (B < 1 || N < 1 || H < 1) return fail(S2_ERR_SHAPE, "B, N, H must be positive");
  if (D != 64 && D != 128) return fail(S2_ERR_UNSUPPORTED, "D=%lld: the prologue supports D in {64, 128}", (long long)D);
  if (B * N >= (int64_t(1) << 31) || B * N * H * D >= (int64_t(1) << 62)) return fail(S2_ERR_UNSUPPORTED, "too large");
  if (!(base > 1.0) || !(scale > 0.0)) return fail(S2_ERR_INVALID_ARG, "base must be > 1 and scale > 0");
  if (!q || !k || !q_out || !k_out) return fail(S2_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out) ||
      (reinterpret_cast<uintptr_t>(positions) & 3u))
    return fail(S2_ERR_INVALID_ARG, "q, k, q_out, k_out must be 16-byte aligned (positions 4-byte)");
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  return launch_status(s2::launch_rope(q, k, q_out, k_out, positions, (int)B, (int)N, (int)H, (int)D, base, scale,
                                       static_cast<cudaStream_t>(stream)),
                       "rope");
}

int s2attn_doc_bounds(const int32_t* doc_ids, int32_t* doc_bounds, int64_t B, int64_t N, void* stream) {
  if (B < 1 || N < 1) return fail(S2_ERR_SHAPE, "B=%lld and N=%lld must be positive", (long long)B, (long long)N);
  if (B * N >= (int64_t(1) << 30)) return fail(S2_ERR_UNSUPPORTED, "B*N must be below 2^30");
  if (!doc_ids || !doc_bounds) return fail(S2_ERR_INVALID_ARG, "null pointer argument");
  if ((reinterpret_cast<uintptr_t>(doc_ids) & 3u) || (reinterpret_cast<uintptr_t>(doc_bounds) & 7u))
    return fail(S2_ERR_INVALID_ARG, "doc_ids must be 4-byte and doc_bounds 8-byte aligned");
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  return launch_status(s2::launch_doc_bounds(doc_ids, doc_bounds, (int)B, (int)N, static_cast<cudaStream_t>(stream)),
                       "document bounds");
}

// Workspace = [-Delta: B*H*N f32][-lse*log2(e): B*H*N f32], each part starting
// on a 256-byte boundary.
static size_t stat_bytes(int64_t B, int64_t N, int64_t H) {
  return ((size_t)B * H * N * sizeof(float) + 255) / 256 * 256;
}

size_t s2attn_bwd_workspace_size(int64_t B, int64_t N, int64_t H, int64_t D) {
  if (B < 1 || N < 1 || H < 1 || D < 1) return 0;
  return 2 * stat_bytes(B, N, H);
}

// Bytes of the stored-dS area: one 128x128 bf16 tile per computed tile pair.
static size_t ds_bytes(const s2::Plan& p) {
  return (size_t)p.B * p.H * (size_t)p.ds_head_tiles * s2::kTile * s2::kTile * 2;
}

// Pointer and workspace checks, tensor maps over [B, plan.N, H, D] and the backward stages.
static int bwd_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, const s2::Plan& plan, void* workspace,
                      size_t workspace_bytes, int stages, void* stream) {
  if (stages < 1 || stages > S2_BWD_ALL_DS || stages == S2_BWD_STORE_DS)
    return fail(S2_ERR_INVALID_ARG, "stages must be a non-empty subset of 7, optionally with S2_BWD_STORE_DS");
  int rc;
  const int64_t B = plan.B, N = plan.N, H = plan.H, D = plan.D;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace)
    return fail(S2_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(S2_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(S2_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const bool stored = (stages & S2_BWD_STORE_DS) != 0;
  const size_t stats = s2attn_bwd_workspace_size(B, N, H, D);
  const size_t need = stats + (stored ? ds_bytes(plan) : 0);
  if (workspace_bytes < need)
    return fail(S2_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes, need);

  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq;
  if ((rc = make_tmap(st, &tq, q, B, N, H, D)) || (rc = make_tmap(st, &tk, k, B, N, H, D)) ||
      (rc = make_tmap(st, &tv, v, B, N, H, D)) || (rc = make_tmap(st, &tdo, dout, B, N, H, D)) ||
      (rc = make_tmap(st, &tdk, dk, B, N, H, D)) || (rc = make_tmap(st, &tdv, dv, B, N, H, D)) ||
      (rc = make_tmap(st, &tdq, dq, B, N, H, D)))
    return rc;
  s2::BwdArgs a;
  a.tmQ = &tq; a.tmK = &tk; a.tmV = &tv; a.tmdO = &tdo; a.tmdK = &tdk; a.tmdV = &tdv; a.tmdQ = &tdq;
  a.plan = plan;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  const size_t sb = stat_bytes(B, N, H);
  a.delta = static_cast<float*>(workspace);
  a.lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + sb);
  // stored dS: bf16 tiles of 32 KB after the row statistics (bulk copies need 16-byte alignment)
  a.ds = stored ? static_cast<char*>(workspace) + stats : nullptr;
  a.status = st->status;
  a.stream = static_cast<cudaStream_t>(stream);
  return launch_status(s2::launch_bwd(a, stages), "backward");
}

size_t s2attn_bwd_ds_workspace_size(int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int variant) {
  if (validate(B, N, H, D, G, N, variant) != S2_OK) return 0;
  const s2::Plan p = s2::make_plan((int)B, (int)N, (int)H, (int)D, (int)G, (int)N, variant);
  return s2attn_bwd_workspace_size(B, N, H, D) + ds_bytes(p);
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, const int32_t* docs, void* dq, void* dk, void* dv, int64_t B, int64_t N,
                    int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant, void* workspace,
                    size_t workspace_bytes, int stages, void* stream) {
  if (stages < 1 || stages > S2_BWD_ALL_DS || stages == S2_BWD_STORE_DS)
    return fail(S2_ERR_INVALID_ARG, "stages must be a non-empty subset of 7, optionally with S2_BWD_STORE_DS");
  int rc = validate(B, N, H, D, G, n_valid, variant);
  if (rc) return rc;
  s2::Plan plan = s2::make_plan((int)B, (int)N, (int)H, (int)D, (int)G, (int)n_valid, variant);
  plan.docs = docs;
  return bwd_launch(q, k, v, o, dout, lse, dq, dk, dv, plan, workspace, workspace_bytes, stages, stream);
}

// ------------------------------------------------------------ sequence parallelism

// Shape rules of one rank's call: the method's rules on the shard (L a
// multiple of G), padding only on the last rank, ROLLED without padding.
static int validate_sp(int64_t B, int64_t L, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                       int rank, int world) {
  if (variant != S2_STRICT && variant != S2_ROLLED)
    return fail(variant == S2_DENSE_CAUSAL ? S2_ERR_UNSUPPORTED : S2_ERR_INVALID_ARG,
                "sequence parallelism supports the STRICT and ROLLED variants (got %d)", variant);
  if (world < 1 || rank < 0 || rank >= world)
    return fail(S2_ERR_INVALID_ARG, "rank %d out of range for world %d", rank, world);
  int rc = validate(B, L, H, D, G, n_valid, variant);
  if (rc) return rc;
  if (n_valid < L && rank != world - 1)
    return fail(S2_ERR_SHAPE, "only the last rank may hold padding (rank %d of %d, n_valid %lld < L %lld)", rank,
                world, (long long)n_valid, (long long)L);
  if (variant == S2_ROLLED && n_valid < L)
    return fail(S2_ERR_UNSUPPORTED, "ROLLED across ranks needs an unpadded sequence");
  if (B * (L + G / 2) >= (int64_t(1) << 31) || B * H * (L + G / 2) >= (int64_t(1) << 31))
    return fail(S2_ERR_UNSUPPORTED, "B*(L+G/2) and B*H*(L+G/2) must be below 2^31");
  return S2_OK;
}

static s2::Plan plan_sp(int64_t B, int64_t L, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                        int rank) {
  return s2::make_plan_sp((int)B, (int)L, (int)H, (int)D, (int)G, (int)(G / 2 + n_valid),
                          variant == S2_STRICT && rank == 0);
}

int s2attn_sp_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t L,
                  int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant, int rank, int world, void* stream) {
  int rc = validate_sp(B, L, H, D, G, n_valid, variant, rank, world);
  if (rc) return rc;
  return fwd_launch(q, k, v, o, lse, plan_sp(B, L, H, D, G, n_valid, variant, rank), stream);
}

int s2attn_sp_bwd_stages(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t L, int64_t H, int64_t D,
                         int64_t G, int64_t n_valid, int variant, int rank, int world, void* workspace,
                         size_t workspace_bytes, int stages, void* stream) {
  int rc = validate_sp(B, L, H, D, G, n_valid, variant, rank, world);
  if (rc) return rc;
  return bwd_launch(q, k, v, o, dout, lse, dq, dk, dv, plan_sp(B, L, H, D, G, n_valid, variant, rank), workspace,
                    workspace_bytes, stages, stream);
}

int s2attn_sp_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, int64_t B, int64_t L, int64_t H, int64_t D, int64_t G,
                  int64_t n_valid, int variant, int rank, int world, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return s2attn_sp_bwd_stages(q, k, v, o, dout, lse, dq, dk, dv, B, L, H, D, G, n_valid, variant, rank, world,
                              workspace, workspace_bytes, S2_BWD_ALL, stream);
}

size_t s2attn_sp_ds_workspace_size(int64_t B, int64_t L, int64_t H, int64_t D, int64_t G, int variant, int rank,
                                   int world) {
  if (validate_sp(B, L, H, D, G, L, variant, rank, world) != S2_OK) return 0;
  const s2::Plan p = plan_sp(B, L, H, D, G, L, variant, rank);
  return s2attn_bwd_workspace_size(B, G / 2 + L, H, D) + ds_bytes(p);
}

size_t s2attn_sp_halo_bytes(int64_t B, int64_t H, int64_t D, int64_t G) {
  if (B < 1 || H < 2 || D < 1 || G < 2) return 0;
  return (size_t)(2 * B * (G / 2) * (H / 2) * D * 2);
}

static int halo_impl(void* a, void* b, void* msg, int64_t B, int64_t L, int64_t H, int64_t D, int64_t G, int part,
                     bool pack, void* stream) {
  if (part != S2_SP_KV && part != S2_SP_GRAD) return fail(S2_ERR_INVALID_ARG, "part must be S2_SP_KV or S2_SP_GRAD");
  int rc = validate(B, L, H, D, G, L, S2_STRICT);
  if (rc) return rc;
  if (!a || !b || !msg) return fail(S2_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(a) || !aligned16(b) || !aligned16(msg))
    return fail(S2_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  return launch_status(s2::launch_halo(a, b, msg, (int)B, (int)L, (int)H, (int)D, (int)G, part, pack,
                                       static_cast<cudaStream_t>(stream)),
                       "halo");
}

int s2attn_sp_halo_pack(const void* a, const void* b, void* msg, int64_t B, int64_t L, int64_t H, int64_t D,
                        int64_t G, int part, void* stream) {
  return halo_impl(const_cast<void*>(a), const_cast<void*>(b), msg, B, L, H, D, G, part, true, stream);
}

int s2attn_sp_halo_unpack(const void* msg, void* a, void* b, int64_t B, int64_t L, int64_t H, int64_t D, int64_t G,
                          int part, void* stream) {
  return halo_impl(a, b, const_cast<void*>(msg), B, L, H, D, G, part, false, stream);
}

int s2attn_bwd_stages_v(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H, int64_t D,
                        int64_t G, int64_t n_valid, int variant, void* workspace, size_t workspace_bytes,
                        int stages, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, nullptr, dq, dk, dv, B, N, H, D, G, n_valid, variant, workspace,
                  workspace_bytes, stages, stream);
}

int s2attn_bwd_docs(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                    const int32_t* doc_bounds, void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H,
                    int64_t D, int64_t G, int64_t n_valid, int variant, void* workspace, size_t workspace_bytes,
                    int stages, void* stream) {
  if (!doc_bounds) return fail(S2_ERR_INVALID_ARG, "null doc_bounds (use s2attn_bwd_stages_v without documents)");
  if (reinterpret_cast<uintptr_t>(doc_bounds) & 7u) return fail(S2_ERR_INVALID_ARG, "doc_bounds must be 8-byte aligned");
  return bwd_impl(q, k, v, o, dout, lse, doc_bounds, dq, dk, dv, B, N, H, D, G, n_valid, variant, workspace,
                  workspace_bytes, stages, stream);
}

int s2attn_bwd_v(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H, int64_t D, int64_t G,
                 int64_t n_valid, int variant, void* workspace, size_t workspace_bytes, void* stream) {
  return s2attn_bwd_stages_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, n_valid, variant, workspace,
                             workspace_bytes, S2_BWD_ALL, stream);
}

int s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int variant,
               void* workspace, size_t workspace_bytes, void* stream) {
  return s2attn_bwd_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, N, variant, workspace, workspace_bytes,
                      stream);
}

static int adjacency_impl(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                          const int32_t* doc_bounds, int format, void* out, void* stream) {
  // D does not enter the pattern; validate with a supported D.
  int rc = validate(1, N, 2, 128, G, n_valid, variant);
  if (rc) return rc;
  if (head_class != 0 && head_class != 1) return fail(S2_ERR_INVALID_ARG, "head_class must be 0 or 1");
  if (format != 0 && format != 1) return fail(S2_ERR_INVALID_ARG, "format must be 0 (bits) or 1 (intervals)");
  if (format == 0 && N > 65536) return fail(S2_ERR_UNSUPPORTED, "bit format supports N <= 65536");
  if (!out) return fail(S2_ERR_INVALID_ARG, "null output pointer");
  if (!aligned16(out)) return fail(S2_ERR_INVALID_ARG, "output must be 16-byte aligned");
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  s2::Plan p = s2::make_plan(1, (int)N, 2, 128, (int)G, (int)n_valid, variant);
  p.docs = doc_bounds;
  const int cls = (variant == S2_DENSE_CAUSAL) ? 0 : head_class;
  return launch_status(s2::launch_adjacency(p, cls, format, out, static_cast<cudaStream_t>(stream)), "adjacency");
}

int s2attn_debug_adjacency(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class, int format,
                           void* out, void* stream) {
  return adjacency_impl(N, G, n_valid, variant, head_class, nullptr, format, out, stream);
}

int s2attn_debug_adjacency_docs(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                                const int32_t* doc_bounds, int format, void* out, void* stream) {
  if (!doc_bounds) return fail(S2_ERR_INVALID_ARG, "null doc_bounds (use s2attn_debug_adjacency without documents)");
  if (reinterpret_cast<uintptr_t>(doc_bounds) & 7u) return fail(S2_ERR_INVALID_ARG, "doc_bounds must be 8-byte aligned");
  return adjacency_impl(N, G, n_valid, variant, head_class, doc_bounds, format, out, stream);
}

int s2attn_debug_wait_probe(int64_t budget_cycles, void* stream) {
  if (budget_cycles < 1000 || budget_cycles > 4000000000LL)
    return fail(S2_ERR_INVALID_ARG, "budget of %lld cycles outside [1000, 4e9]", (long long)budget_cycles);
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  return launch_status(s2::launch_wait_probe(st->status, (long long)budget_cycles, static_cast<cudaStream_t>(stream)),
                       "wait probe");
}

int s2attn_debug_bounds_probe(int64_t value, int64_t lo, int64_t hi, void* stream) {
  if (lo > hi) return fail(S2_ERR_INVALID_ARG, "bounds probe: lower bound %lld above upper %lld", (long long)lo,
                           (long long)hi);
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  return launch_status(s2::launch_bounds_probe(st->status, (long long)value, (long long)lo, (long long)hi,
                                               static_cast<cudaStream_t>(stream)),
                       "bounds probe");
}

// The status area after the stream's work (synchronises the stream).
static int read_status(void* stream, int (&area)[s2::kStatusInts]) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(S2_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  e = cudaMemcpy(area, st->status, sizeof area, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(S2_ERR_CUDA, "reading the status area: %s", cudaGetErrorString(e));
  return S2_OK;
}

int s2attn_check_status(void* stream) {
  int area[s2::kStatusInts];
  int rc = read_status(stream, area);
  if (rc) return rc;
  const int flags = area[0];
  if (!flags) return S2_OK;
  DeviceState* st = nullptr;
  device_state(&st);
  const int zero[s2::kStatusInts] = {};
  cudaMemcpy(st->status, zero, sizeof zero, cudaMemcpyHostToDevice);
  if (flags & s2::kBoundsFlag) {
    const long long* r = reinterpret_cast<const long long*>(area + 4);
    return fail(S2_ERR_BOUNDS, "bounds check failed at site %d: value %lld outside [%lld, %lld) (flags 0x%x)",
                area[2], r[0], r[1], r[2], flags);
  }
  return fail(S2_ERR_TIMEOUT, "a kernel gave up waiting on a barrier (role flags 0x%x)", flags);
}

int s2attn_debug_bounds_checked(void) { return s2::kBoundsChecked ? 1 : 0; }

int s2attn_debug_bounds_report(int64_t* out, void* stream) {
  if (!out) return fail(S2_ERR_INVALID_ARG, "null output pointer");
  int area[s2::kStatusInts];
  int rc = read_status(stream, area);
  if (rc) return rc;
  const long long* r = reinterpret_cast<const long long*>(area + 4);
  out[0] = area[1] ? area[2] : 0;
  out[1] = area[1] ? r[0] : 0;
  out[2] = area[1] ? r[1] : 0;
  out[3] = area[1] ? r[2] : 0;
  return S2_OK;
}

}  // extern "C"
