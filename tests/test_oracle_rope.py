"""Pins for the float64 RoPE reference (oracle/rope.py).

"4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1.1: rotations read original
position IDs, position interpolation maps p to p·L0/L1, and the rotated Q/K
must not depend on the group size (changing the group ratio with the global
position IDs fixed leaves the rotation unchanged).
"""
from __future__ import annotations

import numpy as np

from oracle import rope

RNG = np.random.default_rng(7)


def _x(B=2, N=37, H=3, D=16):
    return RNG.standard_normal((B, N, H, D))


def test_position_zero_is_identity():
    x = _x()
    pos = np.zeros(x.shape[:2], dtype=np.int64)
    np.testing.assert_array_equal(rope.rope(x, pos), x)


def test_rotation_preserves_each_pair_norm():
    x = _x()
    y = rope.rope(x)
    D = x.shape[-1]
    n_x = x[..., : D // 2] ** 2 + x[..., D // 2:] ** 2
    n_y = y[..., : D // 2] ** 2 + y[..., D // 2:] ** 2
    np.testing.assert_allclose(n_y, n_x, rtol=1e-12)


def test_dot_product_depends_only_on_relative_position():
    D = 32
    q = RNG.standard_normal(D)
    k = RNG.standard_normal(D)

    def score(pq, pk):
        qr = rope.rope(q[None, None, None, :], np.array([[pq]]))[0, 0, 0]
        kr = rope.rope(k[None, None, None, :], np.array([[pk]]))[0, 0, 0]
        return qr @ kr

    for d in (0, 1, 5, 100):
        vals = [score(p + d, p) for p in (0, 3, 17, 4096)]
        np.testing.assert_allclose(vals, vals[0], rtol=1e-9, atol=1e-9)
    # and it does change with the relative position
    assert abs(score(10, 0) - score(0, 0)) > 1e-3


def test_position_interpolation_scales_positions():
    x = _x(B=1, N=8)
    pos = np.array([[0, 1, 2, 3, 4096, 8191, 32767, 99999]])
    np.testing.assert_allclose(rope.rope(x, pos, scale=0.25), rope.rope(x, pos * 0.25), rtol=0, atol=1e-12)


def test_matches_textbook_complex_rotation():
    # (x[k] + i x[k+D/2]) · e^{i a_k}: the rotation written with complex numbers
    x = _x(B=1, N=9, H=2, D=8)
    y = rope.rope(x)
    z = (x[..., :4] + 1j * x[..., 4:]) * np.exp(1j * rope.angles(np.arange(9)[None, :], 8)[:, :, None, :])
    np.testing.assert_allclose(y[..., :4], z.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y[..., 4:], z.imag, rtol=0, atol=1e-12)


def test_rotation_does_not_depend_on_grouping():
    # the prologue takes no group size: the same global positions give the same rotation
    x = _x(B=1, N=64)
    pos = np.arange(64)[None, :]
    a = rope.rope(x, pos)
    # inverse-shifting a shifted copy (roll by G/2 for G = 16) then rotating at the original
    # positions equals rotating first: positions travel with their tokens
    rolled = np.roll(x, -8, axis=1)
    rolled_pos = np.roll(pos, -8, axis=1)
    b = np.roll(rope.rope(rolled, rolled_pos), 8, axis=1)
    np.testing.assert_array_equal(a, b)
