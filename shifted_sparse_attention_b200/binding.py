"""Thin ctypes binding of libs2attn.so (declared in include/s2attn.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or the GPU is not an
sm_100a part, calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
from pathlib import Path

import torch

STRICT, ROLLED, DENSE_CAUSAL = 0, 1, 2
S2_OK, S2_ERR_INVALID_ARG, S2_ERR_SHAPE, S2_ERR_UNSUPPORTED, S2_ERR_CUDA, S2_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
S2_ERR_BOUNDS = -6

LIB_PATH = Path(__file__).resolve().parent / "libs2attn.so"
# the same library with the kernels' bounds checks compiled in (include/s2attn.h)
DEBUG_LIB_PATH = Path(__file__).resolve().parent / "libs2attn_debug.so"

# name -> (argtypes, restype), mirroring include/s2attn.h
_i64, _int, _vp, _fp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "s2attn_fwd": ([_vp, _vp, _vp, _vp, _fp, _i64, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "s2attn_fwd_v": ([_vp, _vp, _vp, _vp, _fp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "s2attn_bwd_workspace_size": ([_i64, _i64, _i64, _i64], _sz),
    "s2attn_bwd_ds_workspace_size": ([_i64, _i64, _i64, _i64, _i64, _int], _sz),
    "s2attn_bwd": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int,
                    _vp, _sz, _vp], _int),
    "s2attn_bwd_v": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64,
                      _int, _vp, _sz, _vp], _int),
    "s2attn_bwd_stages_v": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64,
                             _int, _vp, _sz, _int, _vp], _int),
    "s2attn_bwd_noalloc_v": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64,
                              _int, _vp], _int),
    "s2attn_doc_bounds": ([_vp, _vp, _i64, _i64, _vp], _int),
    "s2attn_rope": ([_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_double, ctypes.c_double, _vp],
                    _int),
    "s2attn_graph_gap": ([_fp, _fp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _fp, _fp, _fp, _vp], _int),
    "s2attn_fwd_docs": ([_vp, _vp, _vp, _vp, _fp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "s2attn_bwd_docs": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64,
                         _int, _vp, _sz, _int, _vp], _int),
    "s2attn_sp_fwd": ([_vp, _vp, _vp, _vp, _fp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _int, _vp], _int),
    "s2attn_sp_bwd": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int,
                       _int, _vp, _sz, _vp], _int),
    "s2attn_sp_halo_bytes": ([_i64, _i64, _i64, _i64], _sz),
    "s2attn_sp_bwd_stages": ([_vp, _vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int,
                              _int, _int, _vp, _sz, _int, _vp], _int),
    "s2attn_sp_ds_workspace_size": ([_i64, _i64, _i64, _i64, _i64, _int, _int, _int], _sz),
    "s2attn_sp_halo_pack": ([_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "s2attn_sp_halo_unpack": ([_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int, _vp], _int),
    "s2attn_debug_adjacency": ([_i64, _i64, _i64, _int, _int, _int, _vp, _vp], _int),
    "s2attn_debug_adjacency_docs": ([_i64, _i64, _i64, _int, _int, _vp, _int, _vp, _vp], _int),
    "s2attn_check_status": ([_vp], _int),
    "s2attn_debug_bounds_checked": ([], _int),
    "s2attn_debug_bounds_report": ([_vp, _vp], _int),
    "s2attn_debug_bounds_probe": ([_i64, _i64, _i64, _vp], _int),
    "s2attn_debug_wait_probe": ([_i64, _vp], _int),
    "s2attn_last_error": ([], ctypes.c_char_p),
    "s2attn_version": ([], _int),
}

_lib = None


class S2AttnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__("s2attn error %d: %s" % (code, message))
        self.code = code


def _load(path: Path) -> ctypes.CDLL:
    if not path.exists():
        raise ImportError("%s is not built; run `python -m shifted_sparse_attention_b200.build`" % path.name)
    L = ctypes.CDLL(str(path))
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


def lib() -> ctypes.CDLL:
    """Load libs2attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


_debug_lib = None


@contextlib.contextmanager
def debug_library():
    """Route every call of this module through libs2attn_debug.so (the kernels
    with their bounds checks) inside the block."""
    global _lib, _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(DEBUG_LIB_PATH)
    saved = lib()
    _lib = _debug_lib
    try:
        yield _debug_lib
    finally:
        _lib = saved


def bounds_report(stream=None) -> tuple:
    """(site, value, lower, upper) of the first bounds violation the debug build
    recorded on this device, or zeros (include/s2attn.h)."""
    out = (ctypes.c_int64 * 4)()
    _check(lib().s2attn_debug_bounds_report(ctypes.cast(out, ctypes.c_void_p), _stream(stream)))
    return tuple(int(v) for v in out)


def _check(rc: int) -> None:
    if rc != S2_OK:
        raise S2AttnError(rc, lib().s2attn_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ raw entry points (same names as the C ABI)


def s2attn_fwd_v(q, k, v, o, lse, B, N, H, D, G, n_valid, variant, stream=None) -> int:
    return lib().s2attn_fwd_v(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, N, H, D, G, n_valid, variant,
                              _stream(stream))


def s2attn_fwd(q, k, v, o, lse, B, N, H, D, G, variant, stream=None) -> int:
    return lib().s2attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, N, H, D, G, variant, _stream(stream))


def s2attn_bwd_workspace_size(B, N, H, D) -> int:
    return int(lib().s2attn_bwd_workspace_size(B, N, H, D))


def s2attn_bwd_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, n_valid, variant, workspace, workspace_bytes,
                 stream=None) -> int:
    return lib().s2attn_bwd_v(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                              _ptr(dv), B, N, H, D, G, n_valid, variant, _ptr(workspace), workspace_bytes,
                              _stream(stream))


def s2attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, variant, workspace, workspace_bytes,
               stream=None) -> int:
    return lib().s2attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                            _ptr(dv), B, N, H, D, G, variant, _ptr(workspace), workspace_bytes, _stream(stream))


S2_BWD_PREPARE, S2_BWD_DKDV, S2_BWD_DQ, S2_BWD_ALL = 1, 2, 4, 7
S2_BWD_STORE_DS, S2_BWD_ALL_DS = 8, 15


def s2attn_bwd_ds_workspace_size(B, N, H, D, G, variant) -> int:
    return int(lib().s2attn_bwd_ds_workspace_size(B, N, H, D, G, variant))


def s2attn_bwd_stages_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, n_valid, variant, workspace,
                        workspace_bytes, stages, stream=None) -> int:
    return lib().s2attn_bwd_stages_v(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                     _ptr(dk), _ptr(dv), B, N, H, D, G, n_valid, variant, _ptr(workspace),
                                     workspace_bytes, stages, _stream(stream))


def s2attn_bwd_noalloc_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, n_valid, variant, stream=None) -> int:
    """Backward without a caller workspace (fixed library scratch; see include/s2attn.h)."""
    return lib().s2attn_bwd_noalloc_v(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                      _ptr(dk), _ptr(dv), B, N, H, D, G, n_valid, variant, _stream(stream))


def s2attn_doc_bounds(doc_ids, doc_bounds, B, N, stream=None) -> int:
    return lib().s2attn_doc_bounds(_ptr(doc_ids), _ptr(doc_bounds), B, N, _stream(stream))


def s2attn_fwd_docs(q, k, v, o, lse, doc_bounds, B, N, H, D, G, n_valid, variant, stream=None) -> int:
    return lib().s2attn_fwd_docs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(doc_bounds), B, N, H, D, G,
                                 n_valid, variant, _stream(stream))


def s2attn_bwd_docs(q, k, v, o, dout, lse, doc_bounds, dq, dk, dv, B, N, H, D, G, n_valid, variant, workspace,
                    workspace_bytes, stages, stream=None) -> int:
    return lib().s2attn_bwd_docs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(doc_bounds),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, N, H, D, G, n_valid, variant, _ptr(workspace),
                                 workspace_bytes, stages, _stream(stream))


def s2attn_graph_gap(lse_s2, lse_full, o_s2, o_full, B, N, H, D, G, n_valid, variant, rho, dist, stats,
                     stream=None) -> int:
    return lib().s2attn_graph_gap(_ptr(lse_s2), _ptr(lse_full), _ptr(o_s2), _ptr(o_full), B, N, H, D, G, n_valid,
                                  variant, _ptr(rho), _ptr(dist), _ptr(stats), _stream(stream))


def s2attn_rope(q, k, q_out, k_out, positions, B, N, H, D, base, scale, stream=None) -> int:
    return lib().s2attn_rope(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _ptr(positions), B, N, H, D, float(base),
                             float(scale), _stream(stream))


def rope(q, k, positions=None, base: float = 10000.0, scale: float = 1.0, inplace: bool = False, out=None,
         stream=None):
    """Rotary position prologue on original positions (see include/s2attn.h); returns (q', k').
    ``out``: optional preallocated (q_out, k_out); ``inplace`` rotates q and k themselves."""
    B, N, H, D = _shape(q)
    if _shape(k) != (B, N, H, D):
        raise ValueError("q and k must have the same shape")
    if positions is not None and (positions.shape != (B, N) or positions.dtype != torch.int32 or not positions.is_cuda
                                  or not positions.is_contiguous()):
        raise ValueError("positions must be a contiguous CUDA int32 tensor [B, N]")
    if inplace:
        qo, ko = q, k
    elif out is not None:
        qo, ko = out
        if _shape(qo) != (B, N, H, D) or _shape(ko) != (B, N, H, D):
            raise ValueError("out tensors must match q")
    else:
        qo, ko = torch.empty_like(q), torch.empty_like(k)
    _check(s2attn_rope(q, k, qo, ko, positions, B, N, H, D, base, scale, stream))
    return qo, ko


S2_SP_KV, S2_SP_GRAD = 0, 1
def s2attn_sp_fwd(q, k, v, o, lse, B, L, H, D, G, n_valid, variant, rank, world, stream=None) -> int:
    return lib().s2attn_sp_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, L, H, D, G, n_valid, variant, rank,
                               world, _stream(stream))


def s2attn_sp_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, L, H, D, G, n_valid, variant, rank, world, workspace,
                  workspace_bytes, stream=None) -> int:
    return lib().s2attn_sp_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, L, H, D, G, n_valid, variant, rank, world, _ptr(workspace),
                               workspace_bytes, _stream(stream))


def s2attn_sp_bwd_stages(q, k, v, o, dout, lse, dq, dk, dv, B, L, H, D, G, n_valid, variant, rank, world, workspace,
                         workspace_bytes, stages, stream=None) -> int:
    return lib().s2attn_sp_bwd_stages(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                      _ptr(dv), B, L, H, D, G, n_valid, variant, rank, world, _ptr(workspace),
                                      workspace_bytes, stages, _stream(stream))


def s2attn_sp_ds_workspace_size(B, L, H, D, G, variant, rank, world) -> int:
    return int(lib().s2attn_sp_ds_workspace_size(B, L, H, D, G, variant, rank, world))


def s2attn_sp_halo_bytes(B, H, D, G) -> int:
    return int(lib().s2attn_sp_halo_bytes(B, H, D, G))


def s2attn_sp_halo_pack(a, b, msg, B, L, H, D, G, part, stream=None) -> int:
    return lib().s2attn_sp_halo_pack(_ptr(a), _ptr(b), _ptr(msg), B, L, H, D, G, part, _stream(stream))


def s2attn_sp_halo_unpack(msg, a, b, B, L, H, D, G, part, stream=None) -> int:
    return lib().s2attn_sp_halo_unpack(_ptr(msg), _ptr(a), _ptr(b), B, L, H, D, G, part, _stream(stream))


S2_GAP_BUCKETS = 32


def graph_gap(q, k, v, G: int, variant: int = STRICT, n_valid: int | None = None, stream=None):
    """Training / inference graph gap of one attention layer: runs the S² and the
    dense causal forward on the same inputs and returns (rho, dist, stats): per
    row rho = exp(lse_S2 - lse_full) and dist = ||o_S2 - o_full||_2 ([B, H, N]
    float32), and per head class and segment-position bucket the row count,
    mean rho, min rho and mean dist ([2, S2_GAP_BUCKETS, 4])."""
    B, N, H, D = _shape(q)
    nv = N if n_valid is None else int(n_valid)
    o_s, l_s = forward(q, k, v, G, variant, nv, stream=stream)
    o_f, l_f = forward(q, k, v, N, DENSE_CAUSAL, nv, stream=stream)
    rho = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dist = torch.empty_like(rho)
    stats = torch.empty((2, S2_GAP_BUCKETS, 4), dtype=torch.float32, device=q.device)
    _check(s2attn_graph_gap(l_s, l_f, o_s, o_f, B, N, H, D, G, nv, variant, rho, dist, stats, stream))
    return rho, dist, stats


def s2attn_debug_adjacency(N, G, n_valid, variant, head_class, fmt, out, stream=None) -> int:
    return lib().s2attn_debug_adjacency(N, G, n_valid, variant, head_class, fmt, _ptr(out), _stream(stream))


def s2attn_debug_adjacency_docs(N, G, n_valid, variant, head_class, doc_bounds, fmt, out, stream=None) -> int:
    return lib().s2attn_debug_adjacency_docs(N, G, n_valid, variant, head_class, _ptr(doc_bounds), fmt, _ptr(out),
                                             _stream(stream))


def s2attn_check_status(stream=None) -> int:
    return lib().s2attn_check_status(_stream(stream))


def s2attn_last_error() -> str:
    return lib().s2attn_last_error().decode()


# ------------------------------------------------------------------ tensor-level helpers


def _shape(q):
    if q.dim() != 4 or q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous():
        raise ValueError("expected a contiguous CUDA bf16 tensor [B, N, H, D]")
    return tuple(int(x) for x in q.shape)


def doc_bounds(doc_ids, stream=None):
    """Per-position document bounds [B, N, 2] (int32) from document IDs [B, N] (int32, CUDA)."""
    if doc_ids.dim() != 2 or doc_ids.dtype != torch.int32 or not doc_ids.is_cuda or not doc_ids.is_contiguous():
        raise ValueError("expected a contiguous CUDA int32 tensor [B, N] of document IDs")
    B, N = (int(x) for x in doc_ids.shape)
    out = torch.empty((B, N, 2), dtype=torch.int32, device=doc_ids.device)
    _check(s2attn_doc_bounds(doc_ids, out, B, N, stream))
    return out


def _bounds(docs, B, N):
    if docs.shape != (B, N, 2) or docs.dtype != torch.int32 or not docs.is_cuda or not docs.is_contiguous():
        raise ValueError("expected contiguous CUDA int32 document bounds [B, N, 2] (see doc_bounds)")
    return docs


def forward(q, k, v, G: int, variant: int = STRICT, n_valid: int | None = None, out=None, lse=None, stream=None,
            docs=None):
    """S²-Attn forward; returns (o [B,N,H,D] bf16, lse [B,H,N] fp32).

    docs: optional per-position document bounds [B, N, 2] (from doc_bounds) for
    packed sequences."""
    B, N, H, D = _shape(q)
    nv = N if n_valid is None else int(n_valid)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    if docs is None:
        _check(s2attn_fwd_v(q, k, v, o, l, B, N, H, D, G, nv, variant, stream))
    else:
        _check(s2attn_fwd_docs(q, k, v, o, l, _bounds(docs, B, N), B, N, H, D, G, nv, variant, stream))
    return o, l


def backward(q, k, v, o, dout, lse, G: int, variant: int = STRICT, n_valid: int | None = None,
             grads=None, workspace=None, stream=None, stages: int = 7, docs=None, stored_ds: bool = False):
    """S²-Attn backward; returns (dq, dk, dv) bf16 [B,N,H,D].  docs as for forward.
    stored_ds: the dK/dV stage keeps dS and the dQ stage reads it (adds
    S2_BWD_STORE_DS to `stages`; the workspace must then be of
    s2attn_bwd_ds_workspace_size bytes)."""
    B, N, H, D = _shape(q)
    nv = N if n_valid is None else int(n_valid)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = grads
    if stored_ds:
        stages |= S2_BWD_STORE_DS
        ws_bytes = s2attn_bwd_ds_workspace_size(B, N, H, D, G, variant)
    else:
        ws_bytes = s2attn_bwd_workspace_size(B, N, H, D)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    wb = workspace.numel() * workspace.element_size()
    if docs is None:
        _check(s2attn_bwd_stages_v(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, D, G, nv, variant, workspace, wb,
                                   stages, stream))
    else:
        _check(s2attn_bwd_docs(q, k, v, o, dout, lse, _bounds(docs, B, N), dq, dk, dv, B, N, H, D, G, nv, variant,
                               workspace, wb, stages, stream))
    return dq, dk, dv


def debug_adjacency(N: int, G: int, variant: int, head_class: int, n_valid: int | None = None,
                    fmt: int = 0, device="cuda", docs=None):
    """Visited (query, key) pattern of one head class, from the kernels' scheduler.
    docs: optional document bounds [1, N, 2] or [N, 2] (from doc_bounds) of one sequence."""
    nv = N if n_valid is None else int(n_valid)
    if fmt == 0:
        out = torch.empty((N, (N + 31) // 32), dtype=torch.int32, device=device)
    else:
        out = torch.empty((N, 4), dtype=torch.int32, device=device)
    if docs is None:
        _check(s2attn_debug_adjacency(N, G, nv, variant, head_class, fmt, out))
    else:
        _check(s2attn_debug_adjacency_docs(N, G, nv, variant, head_class, _bounds(docs.reshape(1, N, 2), 1, N), fmt,
                                           out))
    return out


def s2attn_debug_bounds_probe(value, lo, hi, stream=None) -> int:
    return lib().s2attn_debug_bounds_probe(value, lo, hi, _stream(stream))


def s2attn_debug_wait_probe(budget_cycles, stream=None) -> int:
    return lib().s2attn_debug_wait_probe(budget_cycles, _stream(stream))


def check_status(stream=None) -> None:
    _check(s2attn_check_status(stream))


class S2Attention(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in libs2attn.so."""

    @staticmethod
    def forward(ctx, q, k, v, G, variant=STRICT, n_valid=None):
        o, lse = forward(q, k, v, G, variant, n_valid)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.cfg = (G, variant, n_valid)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        G, variant, n_valid = ctx.cfg
        dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, G, variant, n_valid)
        return dq, dk, dv, None, None, None


def s2_attention(q, k, v, G: int, variant: int = STRICT, n_valid: int | None = None):
    return S2Attention.apply(q, k, v, G, variant, n_valid)
