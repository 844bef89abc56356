"""Float64 CPU oracle for shifted sparse attention (S²-Attn).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The product path (the package
``shifted_sparse_attention_b200``) never imports it.

Two independent routes to the same result live here:

* ``s2_oracle.c`` (loaded through ctypes): the visibility matrices A^(0), A^(1)
  written straight from the definitions of "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调"
  §1 (b(i) = floor(i/G), b'(i) = floor((i - G/2)/G), wrapped positions
  excluded or rolled), and masked softmax attention with its gradients from
  §3 of the same page.
* ``segment_path.py``: the "official-style" route the same page §1 asks to
  compare against: shift / slice the second half of the heads, reshape into
  groups, plain causal attention per group, inverse shift; gradients by
  autograd.

Parity status: every function here is pinned by tests in
``tests/test_oracle_pins.py`` (worked examples of the pages, closed-form pair
counts, library causal attention, finite differences, the second route).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "s2_oracle.c"
_LIB = _HERE / "libs2oracle.so"

STRICT, ROLLED, DENSE_CAUSAL = 0, 1, 2


def build(force: bool = False) -> Path:
    """Compile the C oracle with gcc (-O2 -fopenmp) next to its source."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(".so.tmp%d" % os.getpid())
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(_SRC), "-o", str(tmp), "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(_LIB))
        i64, u8p, u16p, dp, i64p = (
            ctypes.c_int64,
            ctypes.POINTER(ctypes.c_uint8),
            ctypes.POINTER(ctypes.c_uint16),
            ctypes.POINTER(ctypes.c_double),
            ctypes.POINTER(ctypes.c_int64),
        )
        L.s2o_visible.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int, i64, i64]
        L.s2o_visible.restype = ctypes.c_int
        L.s2o_adjacency.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int, u8p]
        L.s2o_adjacency.restype = None
        L.s2o_adjacency_row.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int, i64, u8p]
        L.s2o_adjacency_row.restype = None
        L.s2o_pair_count.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int]
        L.s2o_pair_count.restype = i64
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.s2o_pair_count_docs.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int, i32p]
        L.s2o_pair_count_docs.restype = i64
        L.s2o_adjacency_docs.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int, i32p, u8p]
        L.s2o_adjacency_docs.restype = None
        L.s2o_adjacency_row_docs.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int, i32p, i64, u8p]
        L.s2o_adjacency_row_docs.restype = None
        L.s2o_attention.argtypes = [u16p, u16p, u16p, u16p, i32p, i64, i64, i64, i64, i64, i64,
                                    ctypes.c_int, i64, i64, i64p, i64, dp, dp, dp, dp, dp]
        L.s2o_attention.restype = ctypes.c_int
        L.s2o_attention_window.argtypes = [u16p, u16p, u16p, u16p, i32p, i64, i64, i64, i64, i64, i64,
                                           ctypes.c_int, i64, i64, i64p, i64, dp, dp, dp, dp, dp]
        L.s2o_attention_window.restype = ctypes.c_int
        L.s2o_num_threads.argtypes = []
        L.s2o_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def visible(N: int, G: int, n_valid: int, variant: int, head_class: int, i: int, j: int) -> bool:
    return bool(lib().s2o_visible(N, G, n_valid, variant, head_class, i, j))


def adjacency(N: int, G: int, n_valid: int, variant: int, head_class: int) -> np.ndarray:
    """Explicit boolean matrix A^(head_class) of shape [N, N] (row i = query)."""
    out = np.zeros((N, N), dtype=np.uint8)
    lib().s2o_adjacency(N, G, n_valid, variant, head_class, _ptr(out, ctypes.c_uint8))
    return out.astype(bool)


def adjacency_row(N: int, G: int, n_valid: int, variant: int, head_class: int, i: int) -> np.ndarray:
    """Row i of A^(head_class) as a boolean vector of length N."""
    out = np.zeros(N, dtype=np.uint8)
    lib().s2o_adjacency_row(N, G, n_valid, variant, head_class, i, _ptr(out, ctypes.c_uint8))
    return out.astype(bool)


def pair_count(N: int, G: int, n_valid: int, variant: int, head_class: int) -> int:
    return int(lib().s2o_pair_count(N, G, n_valid, variant, head_class))


def pair_count_docs(N: int, G: int, n_valid: int, variant: int, head_class: int, doc) -> int:
    """Visible pairs of one head class under a document mask (doc: N per-position IDs)."""
    d = np.ascontiguousarray(np.asarray(doc, dtype=np.int32))
    assert d.shape == (N,)
    return int(lib().s2o_pair_count_docs(N, G, n_valid, variant, head_class, _ptr(d, ctypes.c_int32)))


def adjacency_docs(N: int, G: int, n_valid: int, variant: int, head_class: int, doc) -> np.ndarray:
    """A^(head_class) restricted to same-document pairs (doc: N per-position IDs), [N, N] bool."""
    d = np.ascontiguousarray(np.asarray(doc, dtype=np.int32))
    assert d.shape == (N,)
    out = np.zeros((N, N), dtype=np.uint8)
    lib().s2o_adjacency_docs(N, G, n_valid, variant, head_class, _ptr(d, ctypes.c_int32), _ptr(out, ctypes.c_uint8))
    return out.astype(bool)


def adjacency_row_docs(N: int, G: int, n_valid: int, variant: int, head_class: int, doc, i: int) -> np.ndarray:
    """Row i of adjacency_docs as a boolean vector of length N."""
    d = np.ascontiguousarray(np.asarray(doc, dtype=np.int32))
    assert d.shape == (N,)
    out = np.zeros(N, dtype=np.uint8)
    lib().s2o_adjacency_row_docs(N, G, n_valid, variant, head_class, _ptr(d, ctypes.c_int32), i,
                                 _ptr(out, ctypes.c_uint8))
    return out.astype(bool)


def _docs(doc, B: int, N: int):
    """Per-position document IDs as a contiguous int32 [B, N] array (None: one document)."""
    if doc is None:
        return None
    try:
        import torch

        if isinstance(doc, torch.Tensor):
            doc = doc.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    d = np.ascontiguousarray(np.asarray(doc, dtype=np.int32))
    if d.shape == (N,):
        d = np.ascontiguousarray(np.broadcast_to(d, (B, N)))
    assert d.shape == (B, N), d.shape
    return d


def num_threads() -> int:
    return int(lib().s2o_num_threads())


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 bit array -> contiguous uint16 numpy array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def attention(q, k, v, dout=None, *, G: int, variant: int, n_valid: int | None = None,
              rows: tuple[int, int] | None = None, heads=None, doc=None):
    """Run the oracle.

    q, k, v, dout: bf16 [B, N, H, D] (torch tensors or uint16 bit arrays).
    Returns a dict of float64 arrays: o [B,N,H,D], lse [B,H,N] and, when dout
    is given, dq, dk, dv.  Only rows in ``rows`` (default all) and heads in
    ``heads`` (flattened b*H+h, default all) are computed; entries outside
    are NaN (o, lse, dq) or hold only the processed rows' contributions
    (dk, dv).  ``doc``: per-position document IDs [B, N] or [N] (document
    mask of packed sequences), or None.
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, H, D = qb.shape
    dd = _docs(doc, B, N)
    nv = N if n_valid is None else int(n_valid)
    r0, r1 = (0, N) if rows is None else rows
    o = np.full((B, N, H, D), np.nan)
    lse = np.full((B, H, N), np.nan)
    want_bwd = dout is not None
    gb = _bits(dout) if want_bwd else None
    dq = np.full((B, N, H, D), np.nan) if want_bwd else np.zeros(1)
    dk = np.zeros((B, N, H, D)) if want_bwd else np.zeros(1)
    dv = np.zeros((B, N, H, D)) if want_bwd else np.zeros(1)
    if heads is None:
        hp, nh = None, 0
    else:
        harr = np.ascontiguousarray(np.asarray(heads, dtype=np.int64))
        hp, nh = _ptr(harr, ctypes.c_int64), len(harr)
    rc = lib().s2o_attention(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(gb, ctypes.c_uint16) if want_bwd else None,
        _ptr(dd, ctypes.c_int32) if dd is not None else None,
        B, N, H, D, G, nv, variant, r0, r1, hp, nh,
        _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
        _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError("oracle rejected the arguments (rc=%d)" % rc)
    out = {"o": o, "lse": lse}
    if want_bwd:
        out.update(dq=dq, dk=dk, dv=dv)
    return out


def attention_window(q, k, v, dout=None, *, G: int, variant: int, rows: tuple[int, int], heads,
                     n_valid: int | None = None, doc=None):
    """The oracle on query rows [r0, r1) of the given heads (flattened b*H+h),
    with compact outputs: o, dq, dk, dv [len(heads), r1 - r0, D]; lse
    [len(heads), r1 - r0].  dk / dv hold the contributions of the window's rows
    to the window's keys only (exact for keys whose visible-from rows all lie in
    the window)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, H, D = qb.shape
    nv = N if n_valid is None else int(n_valid)
    r0, r1 = rows
    dd = _docs(doc, B, N)
    harr = np.ascontiguousarray(np.asarray(heads, dtype=np.int64))
    nh, W = len(harr), r1 - r0
    o = np.full((nh, W, D), np.nan)
    lse = np.full((nh, W), np.nan)
    want_bwd = dout is not None
    gb = _bits(dout) if want_bwd else None
    dq = np.full((nh, W, D), np.nan) if want_bwd else np.zeros(1)
    dk = np.zeros((nh, W, D)) if want_bwd else np.zeros(1)
    dv = np.zeros((nh, W, D)) if want_bwd else np.zeros(1)
    rc = lib().s2o_attention_window(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(gb, ctypes.c_uint16) if want_bwd else None,
        _ptr(dd, ctypes.c_int32) if dd is not None else None,
        B, N, H, D, G, nv, variant, r0, r1, _ptr(harr, ctypes.c_int64), nh,
        _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
        _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError("oracle rejected the arguments (rc=%d)" % rc)
    out = {"o": o, "lse": lse}
    if want_bwd:
        out.update(dq=dq, dk=dk, dv=dv)
    return out
