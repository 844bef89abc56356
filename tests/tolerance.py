"""Parity rules shared by the GPU tests.

Forward O: max-abs error <= 1e-2 and mean-abs error <= 1e-3 against the
float64 oracle.  O is stored in bf16, whose half-ulp is 2^-7 at |o| in [2, 4)
and 2^-6 = 0.0156 at |o| in [4, 8): an element can exceed 1e-2 from the
final rounding alone.  Such an element passes only if its error is within
half_ulp_bf16(o_ref) + 1e-3, and the count of those elements is reported.
Gradients dQ, dK, dV: max|x - x_ref| / max|x_ref| <= 1e-2 and
mean|x - x_ref| / max|x_ref| <= 1e-3, per tensor, over valid rows.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX, O_MEAN = 1e-2, 1e-3
G_MAX, G_MEAN = 1e-2, 1e-3
LSE_ABS = 2e-3


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def check_o(o_gpu, o_ref, where: str = "") -> dict:
    o_gpu, o_ref = to_np(o_gpu), np.asarray(o_ref)
    err = np.abs(o_gpu - o_ref)
    over = err > O_MAX
    floor_ok = err <= half_ulp_bf16(o_ref) + 1e-3
    bad = over & ~floor_ok
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()), n_floor=int((over & floor_ok).sum()),
                 storage_floor=float(np.abs(o_ref - o_ref.astype(np.float32).astype(np.float64)).max()))
    assert not bad.any(), "O error %.4g > %.0e at %d elements %s" % (err[bad].max(), O_MAX, bad.sum(), where)
    assert stats["mean_abs"] <= O_MEAN, "O mean-abs error %.4g %s" % (stats["mean_abs"], where)
    return stats


def check_grad(name, g_gpu, g_ref, where: str = "", tensor_max: float | None = None) -> dict:
    """tensor_max: max |x| of the whole gradient tensor when g_* are a sample of it
    (the bound is scaled by the tensor's max-norm); defaults to the sample's own."""
    g_gpu, g_ref = to_np(g_gpu), np.asarray(g_ref)
    scale = np.abs(g_ref).max()
    if tensor_max is not None:
        scale = max(scale, float(tensor_max))
    scale = scale if scale > 0 else 1.0
    err = np.abs(g_gpu - g_ref) / scale
    stats = dict(max_rel=float(err.max()), mean_rel=float(err.mean()))
    assert stats["max_rel"] <= G_MAX, "%s max error %.4g (scaled) %s" % (name, stats["max_rel"], where)
    assert stats["mean_rel"] <= G_MEAN, "%s mean error %.4g (scaled) %s" % (name, stats["mean_rel"], where)
    return stats


def check_lse(lse_gpu, lse_ref, where: str = ""):
    lse_gpu, lse_ref = to_np(lse_gpu), np.asarray(lse_ref)
    inf_ref = np.isneginf(lse_ref)
    assert (np.isneginf(lse_gpu) == inf_ref).all(), "lse -inf pattern differs %s" % where
    fin = ~inf_ref
    if fin.any():
        e = np.abs(lse_gpu[fin] - lse_ref[fin]).max()
        assert e <= LSE_ABS, "lse error %.4g %s" % (e, where)
