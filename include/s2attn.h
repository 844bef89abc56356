/*
 * s2attn.h -- C ABI of libs2attn.so: shifted sparse attention (S²-Attn)
 * forward and backward on NVIDIA B200 (sm_100a).
 *
 * The operation.  "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1
 * ("S²-Attn的计算图") splits the sequence into groups of G tokens and runs
 * causal attention inside each group.  Heads [0, H/2) use the original
 * boundaries b(i) = floor(i/G); heads [H/2, H) shift by s = G/2 and use
 * b'(i) = floor((i - s)/G); the shifted heads' outputs are returned at their
 * original token positions.  Two boundary treatments of the shifted heads are
 * described there and both are provided:
 *   S2_STRICT        separate short first group [0, s) and last group
 *                    [N - s, N); no key from the future is ever visible;
 *   S2_ROLLED        the sequence is rolled left by s and grouped, with the
 *                    in-group triangular mask of the rolled order: the last
 *                    group is [N - s, N) followed by [0, s), so positions
 *                    [0, s) also see [N - s, N);
 *   S2_DENSE_CAUSAL  plain causal attention over [0, N) for every head (the
 *                    inference graph, §2; also the "full, G = N" setting).
 * For query row i with visible set S_i (§3, "稀疏训练与full推理之间的目标偏移"):
 *   o_i   = sum_{j in S_i} softmax_j(scale q_i·k_j) v_j,  scale = 1/sqrt(D)
 *   lse_i = ln sum_{j in S_i} exp(scale q_i·k_j)
 * and the backward gives dq, dk, dv of L = sum_i dout_i·o_i with
 *   dL/dz_ij = a_ij dout_i·(v_j - o_i),  a_ij = exp(scale q_i·k_j - lse_i).
 *
 * Padding (§1): when the true length n_valid is not a multiple of G the
 * caller pads to N (a multiple of G) before calling; group boundaries are
 * those of the padded N.  Positions >= n_valid are never visible as keys;
 * their query rows get o = 0, lse = -inf, and receive no gradient
 * (dq = dk = dv = 0 there).
 *
 * Layout.  q, k, v, o, dout, dq, dk, dv: bfloat16, [B, N, H, D], contiguous
 * (element (b, i, h, d) at ((b*N + i)*H + h)*D + d).  lse: float32 [B, H, N].
 * All are DEVICE pointers on the current CUDA device, 16-byte aligned.
 * Supported on the GPU: D in {64, 128}; for S2_STRICT / S2_ROLLED, G/2 must be
 * a multiple of 128; for S2_DENSE_CAUSAL, N a multiple of 128.  Always: H
 * even, G even, N a multiple of G, 1 <= n_valid <= N, B*N < 2^31.
 *
 * Ownership and threading.  The caller owns every buffer, including the
 * backward workspace (size from s2attn_bwd_workspace_size).  The library
 * allocates no device memory.  Calls are asynchronous on `stream` (a
 * cudaStream_t; NULL = the legacy default stream) and thread-safe.
 *
 * Errors.  Every call returns S2_OK or a negative code.  Argument, shape and
 * support checks happen on the host before anything is enqueued; on such an
 * error nothing was launched.  S2_ERR_CUDA reports a failed launch.  A kernel
 * that waits on a barrier for longer than about two seconds gives up, leaves
 * its outputs undefined and records a timeout that s2attn_check_status()
 * reports as S2_ERR_TIMEOUT.  s2attn_last_error() returns a message for the
 * last non-OK status of the calling thread.
 */
#ifndef S2ATTN_H_
#define S2ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { S2_STRICT = 0, S2_ROLLED = 1, S2_DENSE_CAUSAL = 2 } s2_variant;

enum {
  S2_OK = 0,
  S2_ERR_INVALID_ARG = -1, /* null or misaligned pointer, unknown enum value */
  S2_ERR_SHAPE = -2,       /* H, G, N, n_valid violate the divisibility / range rules */
  S2_ERR_UNSUPPORTED = -3, /* valid for the method but not for these kernels (D, G/2 % 128, GPU) */
  S2_ERR_CUDA = -4,        /* a CUDA runtime call failed */
  S2_ERR_TIMEOUT = -5,     /* a kernel gave up waiting on a barrier */
  S2_ERR_BOUNDS = -6       /* the debug build found an index outside its bounds (see below) */
};

/* Forward.  Writes o [B,N,H,D] (bf16) and lse [B,H,N] (fp32) for all N rows. */
int s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
               int64_t N, int64_t H, int64_t D, int64_t G, int variant, void* stream);

/* Forward with a valid length n_valid <= N (the call above is n_valid = N). */
int s2attn_fwd_v(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                 int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                 void* stream);

/* Bytes of device workspace s2attn_bwd needs: two float32 row statistics
 * ([B,H,N] each, derived from Delta_i = dout_i·o_i and lse_i), each starting on
 * a 256-byte boundary.  D does not enter the size. */
size_t s2attn_bwd_workspace_size(int64_t B, int64_t N, int64_t H, int64_t D);

/* Backward.  Inputs q, k, v, o, dout (bf16), lse (fp32) as produced by the
 * forward with the same B, N, H, D, G, variant (and n_valid).  Writes dq, dk,
 * dv (bf16 [B,N,H,D]).  `workspace` must hold workspace_bytes >=
 * s2attn_bwd_workspace_size(B, N, H, D) bytes, 256-byte aligned; its contents
 * on entry do not matter. */
int s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H,
               int64_t D, int64_t G, int variant, void* workspace, size_t workspace_bytes,
               void* stream);

int s2attn_bwd_v(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H,
                 int64_t D, int64_t G, int64_t n_valid, int variant, void* workspace,
                 size_t workspace_bytes, void* stream);

/* The backward is three launches on `stream`; s2attn_bwd_v runs all of them
 * in order.  Running them one at a time (same arguments, `stages` a bit set)
 * lets a caller time or overlap them separately:
 *   S2_BWD_PREPARE  row statistics from Delta_i = dout_i·o_i and lse_i, in the
 *                   workspace (reads o, dout, lse);
 *   S2_BWD_DKDV     dk and dv (reads q, k, v, dout and the workspace);
 *   S2_BWD_DQ       dq (reads q, k, v, dout and the workspace).
 * The dk/dv and dq stages are independent of each other; both need the
 * prepare stage of the same call sequence to have run on the same stream
 * with the same workspace.  dq is bitwise reproducible; no stage uses
 * atomic accumulation. */
enum { S2_BWD_PREPARE = 1, S2_BWD_DKDV = 2, S2_BWD_DQ = 4, S2_BWD_ALL = 7 };

/* Stored-dS backward: adding S2_BWD_STORE_DS to `stages` makes the dK/dV
 * stage also write every computed 128x128 tile of dS = P∘(dP − Delta) (bf16)
 * into the workspace, and the dQ stage compute dq = (1/√D)·dS·K from those
 * tiles instead of recomputing S and dP (both stages of one call sequence
 * must carry the flag).  The dQ stage then does no exponentials and a third
 * of the tensor work, and streams the stored tiles from HBM.  The workspace
 * must then hold s2attn_bwd_ds_workspace_size(B, N, H, D, G, variant) bytes
 * (the row statistics plus 32 KB per computed tile pair: about N·G·H·B
 * bytes, 8.7 GB at B1 H32 N32768 G8192).  Results equal the recompute path
 * within rounding (dS is the same bf16 operand; S and dP come from the dK/dV
 * pass's products instead of the dQ pass's own), and are bitwise
 * reproducible run to run. */
enum { S2_BWD_STORE_DS = 8, S2_BWD_ALL_DS = 15 };

size_t s2attn_bwd_ds_workspace_size(int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int variant);

int s2attn_bwd_stages_v(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid,
                        int variant, void* workspace, size_t workspace_bytes, int stages,
                        void* stream);

/* Packed sequences ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1,
 * "因果mask与样本packing"): when several documents are packed into one
 * sequence, key j is visible from query i only if, in addition, both lie in
 * the same document; the same constraint applies to the original and the
 * shifted grouping, so that the shift never puts two documents into one group.
 *
 * The document mask is passed as per-position bounds: doc_bounds is int32
 * [B, N, 2], device memory, 8-byte aligned, entry (b, x) = {first position,
 * one past the last position} of the document holding original position x
 * of batch row b.  Documents must be contiguous runs of positions.
 * s2attn_doc_bounds computes the bounds from per-position document IDs
 * (int32 [B, N]; a document is a maximal run of equal IDs).  Tile pairs that
 * share no document are skipped, so packing many short documents also saves
 * work.  Results are those of s2attn_fwd_v / s2attn_bwd_stages_v with the
 * visibility additionally restricted to same-document pairs. */
int s2attn_doc_bounds(const int32_t* doc_ids, int32_t* doc_bounds, int64_t B, int64_t N, void* stream);

int s2attn_fwd_docs(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int32_t* doc_bounds, int64_t B, int64_t N, int64_t H, int64_t D, int64_t G,
                    int64_t n_valid, int variant, void* stream);

int s2attn_bwd_docs(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, const int32_t* doc_bounds, void* dq, void* dk, void* dv, int64_t B,
                    int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                    void* workspace, size_t workspace_bytes, int stages, void* stream);

/* Rotary position prologue ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1,
 * "RoPE使用原始位置"): Q and K are rotated at each token's ORIGINAL position
 * ID, never its index inside a group, with position interpolation p -> p·scale
 * (scale = L0/L1 when extending a context of L0 tokens to L1).  Pairing:
 * coordinate k with k + D/2 (the Llama convention), angle
 * a_k = (p·scale)·base^(-2k/D):
 *   x'[k] = x[k] cos a_k - x[k+D/2] sin a_k,  x'[k+D/2] = x[k+D/2] cos a_k + x[k] sin a_k.
 * q, k, q_out, k_out: bf16 [B, N, H, D], device, 16-byte aligned; q_out / k_out
 * may equal q / k (in place).  positions: int32 [B, N] original position IDs
 * (e.g. restarting per packed document), or NULL for 0..N-1.  D in {64, 128}.
 * Angles are formed in double precision (they reach 10^5 rad); the rotation
 * is done in float and rounded to bf16. */
int s2attn_rope(const void* q, const void* k, void* q_out, void* k_out, const int32_t* positions,
                int64_t B, int64_t N, int64_t H, int64_t D, double base, double scale, void* stream);

/* Sequence parallelism ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1,
 * "Sequence Parallel通信"): the sequence of N = world·L positions is cut into
 * G-aligned shards, rank r holding original positions [rL, rL + L).  Group
 * boundaries of the unshifted heads then coincide with shard boundaries; the
 * shifted heads' group straddling a boundary needs, on rank r, the s = G/2
 * K/V rows [rL - s, rL) of rank r - 1 (the halo), and returns their partial
 * gradients to it.  Exchanging only this halo (never rolling inside a shard)
 * keeps the multi-rank graph identical to the single-GPU graph.
 *
 * Layout: every tensor of a rank lives in an EXTENDED buffer of s + L rows,
 * [B, s + L, H, D] bf16 (lse [B, H, s + L] fp32), whose rows [0, s) are the
 * halo and rows [s, s + L) the shard.  Halo rows of q, dout are never read;
 * those of o, lse, dq are overwritten with zeros (-inf for lse); those of
 * dk, dv receive the shard's partial gradients of the halo keys.
 *
 * One forward or backward step of a rank:
 *   1. s2attn_sp_halo_pack(k, v, msg, ..., S2_SP_KV): the shard's last s rows
 *      of the shifted heads -> msg (s2attn_sp_halo_bytes bytes); send msg to
 *      rank r + 1 (ROLLED: to (r + 1) mod world; STRICT: the last rank sends
 *      nothing); receive into msg' from rank r - 1 and
 *      s2attn_sp_halo_unpack(msg', k, v, ..., S2_SP_KV) into the halo rows.
 *      (Rank 0 of a STRICT sequence receives nothing; its halo is ignored.)
 *   2. s2attn_sp_fwd / s2attn_sp_bwd on the extended buffers.
 *   3. After the backward: s2attn_sp_halo_pack(dk, dv, msg, ..., S2_SP_GRAD)
 *      sends the halo rows' gradients back to the rank the halo came from,
 *      which adds them with s2attn_sp_halo_unpack(..., S2_SP_GRAD) onto its
 *      last s rows (fp32 sum, one rounding to bf16).
 * With world = 1, ROLLED sends to itself and STRICT sends nothing; both then
 * equal the single-GPU calls.  O, lse and dq of every shard row are bitwise
 * those of the single-GPU call on the whole sequence (same tiles, same order);
 * dk, dv of the s rows in front of each boundary differ by the extra rounding
 * of the two partial sums.
 *
 * Arguments: L = rows of the shard (a multiple of G); n_valid = valid rows of
 * the shard (L except on a padded last rank; ROLLED needs n_valid = L);
 * variant S2_STRICT or S2_ROLLED (S2_DENSE_CAUSAL does not shard this way:
 * S2_ERR_UNSUPPORTED); workspace: s2attn_bwd_workspace_size(B, G/2 + L, H, D)
 * bytes.  The messages are [2][B][s][H/2][D] bf16: V_KV = 2·B·(H/2)·s·D·2
 * bytes per direction, the pages' volume. */
enum { S2_SP_KV = 0, S2_SP_GRAD = 1 };

int s2attn_sp_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t L,
                  int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant, int rank, int world,
                  void* stream);

int s2attn_sp_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t L, int64_t H,
                  int64_t D, int64_t G, int64_t n_valid, int variant, int rank, int world,
                  void* workspace, size_t workspace_bytes, void* stream);

/* The rank backward stage by stage, as s2attn_bwd_stages_v (S2_BWD_STORE_DS
 * included: the workspace must then hold s2attn_sp_ds_workspace_size bytes). */
int s2attn_sp_bwd_stages(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, int64_t B, int64_t L, int64_t H,
                         int64_t D, int64_t G, int64_t n_valid, int variant, int rank, int world,
                         void* workspace, size_t workspace_bytes, int stages, void* stream);

size_t s2attn_sp_ds_workspace_size(int64_t B, int64_t L, int64_t H, int64_t D, int64_t G, int variant,
                                   int rank, int world);

size_t s2attn_sp_halo_bytes(int64_t B, int64_t H, int64_t D, int64_t G);

int s2attn_sp_halo_pack(const void* a, const void* b, void* msg, int64_t B, int64_t L, int64_t H,
                        int64_t D, int64_t G, int part, void* stream);

int s2attn_sp_halo_unpack(const void* msg, void* a, void* b, int64_t B, int64_t L, int64_t H,
                          int64_t D, int64_t G, int part, void* stream);

/* Training / inference graph gap ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调"
 * §3 "稀疏训练与full推理之间的目标偏移", §2.1 diagnostics).  Training normalises
 * row i's softmax over its S² set S_i, inference over its full causal history
 * F_i; when the graph switches, every in-group weight is scaled by
 * Z_s / (Z_s + Z_out).  From two forwards on the same q, k, v -- `variant`
 * (strict or rolled: lse_s2, o_s2) and S2_DENSE_CAUSAL with the same n_valid
 * (lse_full, o_full) -- this writes, per row (float32 [B, H, N]):
 *   rho[b,h,i]  = exp(lse_s2 - lse_full)   (= Z_s / (Z_s + Z_out) for strict),
 *   dist[b,h,i] = || o_s2[b,i,h,:] - o_full[b,i,h,:] ||_2,
 * both 0 on padded rows, and per head class c (0: heads [0,H/2), 1: the
 * shifted heads) and bucket k = floor(log2(l + 1)) of the row's position l
 * inside its S² segment, stats[c][k][0..3] = {row count, mean rho, min rho,
 * mean dist} (float32 [2][S2_GAP_BUCKETS][4], deterministic).  Device
 * pointers; o in the layout of the forward. */
#define S2_GAP_BUCKETS 32
int s2attn_graph_gap(const float* lse_s2, const float* lse_full, const void* o_s2, const void* o_full,
                     int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid, int variant,
                     float* rho, float* dist, float* stats, void* stream);

/* Size of the fixed scratch array behind s2attn_bwd_noalloc_v (32 MiB). */
#define S2_NOALLOC_SCRATCH_BYTES (32u << 20)

/* The backward (same arguments and results as s2attn_bwd_v) for callers that
 * cannot allocate device memory, such as a plug-in inside a framework that
 * owns the device heap, or a runtime held to a fixed memory footprint.  The
 * pages describe no such entry point; it exists for those callers only.
 * Instead of a caller-provided workspace it uses one file-scope device array
 * of S2_NOALLOC_SCRATCH_BYTES.  Shapes whose s2attn_bwd_workspace_size()
 * exceeds that size are rejected with S2_ERR_UNSUPPORTED before anything is
 * launched.
 * When the array is reserved: the driver reserves it when it loads the
 * array's device module into a context, which under CUDA's default lazy
 * module loading happens inside the FIRST call on each device (under
 * CUDA_MODULE_LOADING=EAGER, when the context is created); it stays reserved
 * until that context is destroyed.  A caller whose framework will claim the
 * device heap should make one call at start-up, before the framework
 * reserves its memory and outside any stream capture.  If the device has no
 * room for the array at that first call, the call returns S2_ERR_CUDA with
 * the driver's out-of-memory message and launches nothing.
 * The first call on each device, with that device current, looks up the
 * array's device address and caches it with the identity of the current
 * context; a call in a later context of the device (after cudaDeviceReset)
 * looks it up again.  All calls share the one array: calls whose kernels
 * overlap on the GPU (other streams, other host threads) race on it.  No
 * allocating routine is called by the library itself; every call rewrites
 * the statistics it reads before reading them. */
int s2attn_bwd_noalloc_v(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid,
                         int variant, void* stream);

/* Debug: the (query, key) pairs the kernels visit for one head class
 * (0: heads [0,H/2), 1: heads [H/2,H); ignored for S2_DENSE_CAUSAL), computed
 * by the same scheduler and masks as the forward/backward kernels.
 *   format 0: bitset, uint32 [N][ceil(N/32)], bit j of row i set iff key j is
 *             visited from query i (N <= 65536);
 *   format 1: int32 [N][4] = {lo1, hi1, lo2, hi2}, the visited keys as at most
 *             two inclusive intervals of original positions, -1 when absent.
 * `out` is a device pointer the caller sized accordingly. */
int s2attn_debug_adjacency(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                           int format, void* out, void* stream);

/* Debug: the same dump under a document mask (packed sequences, see
 * s2attn_doc_bounds): the pairs the document-aware kernels visit for one
 * sequence.  doc_bounds is int32 [N, 2] of that sequence (device memory,
 * 8-byte aligned), as s2attn_doc_bounds writes it for B = 1.  A row's
 * visited keys are still at most two intervals in format 1. */
int s2attn_debug_adjacency_docs(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                                const int32_t* doc_bounds, int format, void* out, void* stream);

/* Synchronizes `stream` and reports (then clears) a kernel timeout, or a
 * bounds violation of the debug build, recorded on the current device since
 * the last check: S2_OK, S2_ERR_TIMEOUT or S2_ERR_BOUNDS (the latter first). */
int s2attn_check_status(void* stream);

/* Bounds-checked build.  The library can also be built as
 * libs2attn_debug.so (the same sources with -DS2_DEBUG_BOUNDS): there, before
 * every access, each kernel checks the tile origins it computes against [0, N)
 * and against the rows that may hold them (query tiles [q_begin, n_valid),
 * key tiles [k_begin, n_valid) of the plan), its TMA row coordinates against
 * the tensor, the global indices it stores to, the stored-dS slots against the
 * workspace, and the TMEM columns it addresses against the 512 allocated.
 * The first violation on the device is recorded (site, value, bounds); the
 * access is skipped and the kernel gives up as on a timeout, without a trap,
 * so the context stays usable.  Results of the debug build equal the normal
 * build's bit for bit.
 * s2attn_debug_bounds_checked: 1 in the debug build, 0 in the normal one.
 * s2attn_debug_bounds_report: synchronizes `stream` and writes the first
 * recorded violation as out[4] = {site, value, lower bound (inclusive), upper
 * bound (exclusive)}, or zeros if there is none; it does not clear the record
 * (s2attn_check_status does).  Sites: 1-4 forward (Q tile, K/V tile, output
 * row or lse index, TMEM), 5-9 dK/dV pass (K/V tile, Q/dO tile or statistics
 * rows, stored-dS slot, output row, TMEM), 10-13 dQ passes (Q/dO tile or
 * statistics, K/V tile or stored-dS slot, output row, TMEM), 14 the probe
 * below.
 * s2attn_debug_bounds_probe: launches one thread that runs the same check on
 * `value` against [lo, hi) with site 14 and touches no memory on its result,
 * so the recording path can be exercised without a real violation.  In the
 * normal build the check is compiled out and nothing is recorded.  Returns
 * S2_ERR_INVALID_ARG if lo > hi. */
int s2attn_debug_bounds_checked(void);
int s2attn_debug_bounds_report(int64_t* out, void* stream);
int s2attn_debug_bounds_probe(int64_t value, int64_t lo, int64_t hi, void* stream);

/* Failure-detection probe: launches one CTA whose wait on a barrier that
 * nothing completes runs out after `budget_cycles` SM clocks (in [1000, 4e9]);
 * the kernel records the timeout in the status word (flag 0x200) and exits
 * normally, so the next s2attn_check_status() returns S2_ERR_TIMEOUT and the
 * context stays usable.  It exercises, without any fault, the path every
 * kernel takes when one of its bounded waits gives up. */
int s2attn_debug_wait_probe(int64_t budget_cycles, void* stream);

/* Message for the last non-OK status returned to the calling thread. */
const char* s2attn_last_error(void);

/* ABI version of this header (major*100 + minor): 201. */
int s2attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H_ */
