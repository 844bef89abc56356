"""Float64 reference for the rotary position prologue (RoPE on original positions).

TEST INFRASTRUCTURE ONLY (imported by ``tests/`` and ``bench.py``'s CPU leg;
never by the product package).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1 ("RoPE使用原始位置"): the
shift only permutes tensors, so the rotation reads each token's ORIGINAL
position ID, never its index inside a group; context extension adds position
interpolation, mapping a target position p to p·L0/L1 before the rotation
angles are computed.  The pages do not fix the pairing of coordinates; the
reading taken here is the convention of the Llama models the pages fine-tune:
coordinate k is paired with k + D/2, with angle (p·s)·θ_k,
θ_k = base^(-2k/D), k < D/2, s the interpolation factor:
    x'[k]       = x[k] cos(a_k) - x[k + D/2] sin(a_k)
    x'[k + D/2] = x[k + D/2] cos(a_k) + x[k] sin(a_k)

Parity status: pinned in ``tests/test_oracle_rope.py`` (identity at p = 0,
norm preservation, the relative-position property, the interpolation
identity, independence from the grouping).
"""
from __future__ import annotations

import numpy as np


def angles(positions, D: int, base: float = 10000.0, scale: float = 1.0) -> np.ndarray:
    """a[..., k] = positions·scale·base^(-2k/D), float64, shape positions.shape + (D/2,)."""
    k = np.arange(D // 2, dtype=np.float64)
    theta = base ** (-2.0 * k / D)
    return (np.asarray(positions, dtype=np.float64) * scale)[..., None] * theta


def rope(x, positions=None, *, base: float = 10000.0, scale: float = 1.0) -> np.ndarray:
    """Rotate x [B, N, H, D] (float64 or a bf16 torch tensor) at original positions
    [B, N] (default 0..N-1).  Returns float64 [B, N, H, D]."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().to(torch.float64).cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x, dtype=np.float64)
    B, N, H, D = x.shape
    if positions is None:
        positions = np.broadcast_to(np.arange(N), (B, N))
    a = angles(positions, D, base, scale)[:, :, None, :]  # [B, N, 1, D/2]
    c, s = np.cos(a), np.sin(a)
    lo, hi = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)
