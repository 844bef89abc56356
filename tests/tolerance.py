"""Parity rules shared by the GPU tests.

Forward O: max-abs error <= 1e-2 and mean-abs error <= 1e-3 against the
float64 oracle.  O is stored in bf16, whose half-ulp is 2^-7 at |o| in [2, 4)
and 2^-6 = 0.0156 at |o| in [4, 8): an element can exceed 1e-2 from the
final rounding alone.  Such an element passes only if its error is within
half_ulp_bf16(o_ref) + 1e-3; it is counted (``n_floor``) and reported beside
the storage floor max|bf16(o_ref) - o_ref| at the end of the session, never
passed silently.
Gradients dQ, dK, dV: max|x - x_ref| / max|x_ref| <= 1e-2 and
mean|x - x_ref| / max|x_ref| <= 1e-3, per tensor, over valid rows.  The
scale max|x_ref| always comes from oracle values: a test that checks a
sample of a tensor passes the oracle's maximum over every sample it
computed, never a value read from the CUDA output.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

O_MAX, O_MEAN = 1e-2, 1e-3
G_MAX, G_MEAN = 1e-2, 1e-3
# lse has no stated tolerance; this one follows from the kernel's arithmetic.  The
# forward's row sum l adds the softmax weights after their rounding to bf16 (so
# that o stays a convex combination of the v_j), and round-to-nearest-even to
# bf16's 8 significant bits changes each weight by at most 2^-8 of its value.  A
# sum of such weights is off by at most 2^-8 relative, so ln l by at most
# ln(1 + 2^-8) = 3.90e-3; the fp32 scores (D bf16 products accumulated in fp32,
# times 1/sqrt(D)) and the approximate exp2 / log2 add well under 1e-4.
LSE_ABS = math.log1p(2.0 ** -8) + 1e-4

# One record per check_o call: the test it ran in (set by an autouse fixture in
# conftest.py), where, the errors, the storage floor and how many elements passed
# on the bf16 allowance alone.  Printed at the end of the session and, when the
# environment names a file in S2_PARITY_REPORT, appended there as JSON lines.
CURRENT_TEST = ""
O_RECORDS: list[dict] = []


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (8 significant bits, ties to
    even) in one step, without passing through float32."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def storage_floor(o_ref: np.ndarray) -> float:
    """Largest error a bf16 output can have from its final rounding alone."""
    o_ref = np.asarray(o_ref, dtype=np.float64)
    fin = np.isfinite(o_ref)
    if not fin.any():
        return 0.0
    return float(np.abs(bf16_rne(o_ref[fin]) - o_ref[fin]).max())


def _record(rec: dict) -> None:
    rec["test"] = CURRENT_TEST
    O_RECORDS.append(rec)
    path = os.environ.get("S2_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def check_o(o_gpu, o_ref, where: str = "") -> dict:
    o_gpu, o_ref = to_np(o_gpu), np.asarray(o_ref)
    err = np.abs(o_gpu - o_ref)
    over = err > O_MAX
    floor_ok = err <= half_ulp_bf16(o_ref) + 1e-3
    bad = over & ~floor_ok
    stats = dict(where=where, max_abs=float(err.max()), mean_abs=float(err.mean()),
                 n_floor=int((over & floor_ok).sum()), n_elems=int(err.size),
                 storage_floor=storage_floor(o_ref))
    _record(dict(stats))
    assert not bad.any(), "O error %.4g > %.0e at %d elements %s" % (err[bad].max(), O_MAX, bad.sum(), where)
    assert stats["mean_abs"] <= O_MEAN, "O mean-abs error %.4g %s" % (stats["mean_abs"], where)
    return stats


def check_grad(name, g_gpu, g_ref, where: str = "", ref_max: float | None = None) -> dict:
    """ref_max: max |x_ref| of the oracle over every sample of this tensor the
    test computed, when g_ref is one of several samples (the bound is scaled by
    the tensor's max-norm); defaults to the sample's own oracle maximum."""
    g_gpu, g_ref = to_np(g_gpu), np.asarray(g_ref)
    scale = float(np.abs(g_ref).max()) if ref_max is None else float(ref_max)
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


def o_summary() -> list[str]:
    """One line per test that checked O: elements, worst errors, storage floor,
    and the count of elements that passed on the bf16 allowance."""
    by = {}
    for r in O_RECORDS:
        a = by.setdefault(r["test"], dict(n=0, max_abs=0.0, mean_w=0.0, n_floor=0, floor=0.0))
        a["n"] += r["n_elems"]
        a["max_abs"] = max(a["max_abs"], r["max_abs"])
        a["mean_w"] += r["mean_abs"] * r["n_elems"]
        a["n_floor"] += r["n_floor"]
        a["floor"] = max(a["floor"], r["storage_floor"])
    lines = []
    for t, a in by.items():
        lines.append("%s: O elements %d, max-abs %.3g, mean-abs %.3g, storage floor %.3g, "
                     "passed on the bf16 allowance %d" % (t, a["n"], a["max_abs"], a["mean_w"] / max(a["n"], 1),
                                                          a["floor"], a["n_floor"]))
    return lines
